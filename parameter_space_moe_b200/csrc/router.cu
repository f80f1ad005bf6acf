// Router and dt projection: one warp per token.
//
// Paper: Swimba notes, Method, flowchart node "token router R(X_t)" and key design 1
// (pi_t = softmax(g_t) over the active set K_t).  Per token t:
//   g_t,e  = W_r[e] . X_t                         (fp32 accumulation)
//   K_t    = the k largest g_t,e, largest first, equal values -> lower e
//   pi_t,j = exp(g_{K_j} - g_{K_0}) / sum_j' exp(g_{K_j'} - g_{K_0})
//   dt_t,h = clamp(softplus(W_dt[h] . X_t + b_dt[h]), 1e-3, 0.1)
// The token's X row is staged in shared memory as fp32; each lane owns a strided slice of D and the
// warp reduces every dot product with a fixed xor butterfly, so results are deterministic.
#include "common.cuh"

namespace swimba {

constexpr int kRouterWarps = 8;
constexpr int kMaxE = 64;

template <class T>
__global__ void __launch_bounds__(kRouterWarps * 32)
router_kernel(Dims d, const T* __restrict__ X, const T* __restrict__ Wr, const T* __restrict__ Wdt,
              const float* __restrict__ bdt, int32_t* __restrict__ idx_out, float* __restrict__ w_out,
              float* __restrict__ dt_out) {
  extern __shared__ float xs_all[];  // [warps][D]
  __shared__ float g_s[kRouterWarps][kMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * kRouterWarps + warp;
  if (m >= d.M) return;
  float* xs = xs_all + (size_t)warp * d.D;
  const T* xr = X + (size_t)m * d.D;
  for (int i = lane; i < d.D; i += 32) xs[i] = to_f32(xr[i]);
  __syncwarp();

  for (int e = 0; e < d.E; ++e) {
    const T* wr = Wr + (size_t)e * d.D;
    float acc = 0.f;
    for (int i = lane; i < d.D; i += 32) acc = fmaf(xs[i], to_f32(wr[i]), acc);
    acc = warp_sum(acc);
    if (lane == 0) g_s[warp][e] = acc;
  }
  for (int h = 0; h < d.H; ++h) {
    const T* wr = Wdt + (size_t)h * d.D;
    float acc = 0.f;
    for (int i = lane; i < d.D; i += 32) acc = fmaf(xs[i], to_f32(wr[i]), acc);
    acc = warp_sum(acc) + bdt[h];
    if (lane == 0) {
      float sp = acc > 20.f ? acc : log1pf(expf(acc));
      dt_out[(size_t)m * d.H + h] = fminf(fmaxf(sp, 1e-3f), 0.1f);
    }
  }
  __syncwarp();

  // top-k by k rounds of a warp argmax; lane l holds experts l and l + 32
  float v0 = lane < d.E ? g_s[warp][lane] : -INFINITY;
  float v1 = lane + 32 < d.E ? g_s[warp][lane + 32] : -INFINITY;
  bool taken0 = lane >= d.E, taken1 = lane + 32 >= d.E;
  float gmax = 0.f, sel[8];
  int seli[8];
  for (int j = 0; j < d.k; ++j) {
    // local best (lower index wins ties): lane's expert `lane` precedes `lane + 32`
    float bv; int bi;
    if (!taken0 && (taken1 || v0 >= v1)) { bv = v0; bi = lane; }
    else if (!taken1) { bv = v1; bi = lane + 32; }
    else { bv = -INFINITY; bi = 1 << 30; }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (bi == lane) taken0 = true;
    if (bi == lane + 32) taken1 = true;
    if (j == 0) gmax = bv;
    sel[j] = bv; seli[j] = bi;
  }
  if (lane == 0) {
    float den = 0.f, ex[8];
    for (int j = 0; j < d.k; ++j) { ex[j] = expf(sel[j] - gmax); den += ex[j]; }
    for (int j = 0; j < d.k; ++j) {
      idx_out[(size_t)m * d.k + j] = seli[j];
      w_out[(size_t)m * d.k + j] = ex[j] / den;
    }
  }
}

cudaError_t launch_router(const Dims& d, const void* X, const swimba_weights& w, int32_t* idx, float* wts,
                          float* dt, unsigned* st, cudaStream_t s) {
  (void)st;
  dim3 grid(ceil_div(d.M, kRouterWarps));
  size_t smem = sizeof(float) * (size_t)kRouterWarps * d.D;
  if (d.dtype == SWIMBA_BF16) {
    auto k = router_kernel<__nv_bfloat16>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kRouterWarps * 32, smem, s>>>(d, (const __nv_bfloat16*)X, (const __nv_bfloat16*)w.w_router,
                                             (const __nv_bfloat16*)w.w_dt, w.b_dt, idx, wts, dt);
  } else {
    auto k = router_kernel<float>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kRouterWarps * 32, smem, s>>>(d, (const float*)X, (const float*)w.w_router, (const float*)w.w_dt,
                                             w.b_dt, idx, wts, dt);
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swimba
