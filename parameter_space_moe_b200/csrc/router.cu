// Router and dt projection.
//
// Paper: Swimba notes, Method, flowchart node "token router R(X_t)" and key design 1
// (pi_t = softmax(g_t) over the active set K_t).  Per token t:
//   g_t,e  = W_r[e] . X_t                         (fp32 accumulation)
//   K_t    = the k largest g_t,e, largest first, equal values -> lower e
//   pi_t,j = exp(g_{K_j} - g_{K_0}) / sum_j' exp(g_{K_j'} - g_{K_0})
//   dt_t,h = clamp(softplus(W_dt[h] . X_t + b_dt[h]), 1e-3, 0.1)
// The E + H dot products per token form a skinny GEMM [M x D] x [D x (E + H)].  bf16 layers run it on
// the warp-level tensor-core path (mma.sync m16n8k16, fp32 accumulate), 16 tokens per CTA with the K
// reduction split over 8 warps.  The fp32 layer keeps a CUDA-core kernel (one warp per token, fixed xor
// butterfly reductions).
#include "common.cuh"

namespace swimba {

namespace {
constexpr int kMaxE = 64;

// Top-k, renormalised weights and dt for one token; logits g[0..E) and pre-activations g[E..E+H) in
// (shared) memory, called by a whole warp.
__device__ __forceinline__ void finish_token(const Dims& d, const float* g, const float* __restrict__ bdt, int m,
                                             int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                                             float* __restrict__ dt_out, int32_t* __restrict__ counts) {
  const int lane = threadIdx.x & 31;
  for (int h = lane; h < d.H; h += 32) {
    const float v = g[d.E + h] + bdt[h];
    const float sp = v > 20.f ? v : log1pf(expf(v));
    dt_out[(size_t)m * d.H + h] = fminf(fmaxf(sp, 1e-3f), 0.1f);
  }
  // k rounds of a warp argmax; lane l holds experts l and l + 32 (lower index wins ties)
  float v0 = lane < d.E ? g[lane] : -INFINITY;
  float v1 = lane + 32 < d.E ? g[lane + 32] : -INFINITY;
  bool taken0 = lane >= d.E, taken1 = lane + 32 >= d.E;
  float gmax = 0.f, sel[8];
  int seli[8];
  for (int j = 0; j < d.k; ++j) {
    float bv;
    int bi;
    if (!taken0 && (taken1 || v0 >= v1)) { bv = v0; bi = lane; }
    else if (!taken1) { bv = v1; bi = lane + 32; }
    else { bv = -INFINITY; bi = 1 << 30; }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (bi == lane) taken0 = true;
    if (bi == lane + 32) taken1 = true;
    if (j == 0) gmax = bv;
    sel[j] = bv;
    seli[j] = bi;
  }
  if (lane == 0) {
    float den = 0.f, ex[8];
    for (int j = 0; j < d.k; ++j) { ex[j] = expf(sel[j] - gmax); den += ex[j]; }
    for (int j = 0; j < d.k; ++j) {
      idx_out[(size_t)m * d.k + j] = seli[j];
      w_out[(size_t)m * d.k + j] = ex[j] / den;
      if (counts) atomicAdd(&counts[(size_t)((m * d.k + j) / kDispatchTile) * d.E + seli[j]], 1);
    }
  }
}

// ------------------------------------------------------------------------------------------ CUDA cores
constexpr int kRouterWarps = 8;

template <class T>
__global__ void __launch_bounds__(kRouterWarps * 32)
router_simt_kernel(Dims d, const T* __restrict__ X, const T* __restrict__ Wr, const T* __restrict__ Wdt,
                   const float* __restrict__ bdt, int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                   float* __restrict__ dt_out, int32_t* __restrict__ counts) {
  extern __shared__ float xs_all[];  // [warps][D], then [warps][E + H] logits
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * kRouterWarps + warp;
  if (m >= d.M) return;
  float* xs = xs_all + (size_t)warp * d.D;
  float* g = xs_all + (size_t)kRouterWarps * d.D + (size_t)warp * (d.E + d.H);
  const T* xr = X + (size_t)m * d.D;
  for (int i = lane; i < d.D; i += 32) xs[i] = to_f32(xr[i]);
  __syncwarp();
  for (int r = 0; r < d.E + d.H; ++r) {
    const T* wr = r < d.E ? Wr + (size_t)r * d.D : Wdt + (size_t)(r - d.E) * d.D;
    float acc = 0.f;
    for (int i = lane; i < d.D; i += 32) acc = fmaf(xs[i], to_f32(wr[i]), acc);
    acc = warp_sum(acc);
    if (lane == 0) g[r] = acc;
  }
  __syncwarp();
  finish_token(d, g, bdt, m, idx_out, w_out, dt_out, counts);
}

// ------------------------------------------------------------------------------------------ mma.sync
// A CTA owns one m16 tile of tokens; its 8 warps split the K = D reduction into 8 contiguous ranges and
// load their mma.sync fragments straight from global memory (X rows and the stacked [W_r; W_dt] rows are
// read 16 bytes per row per k-step by 4 lanes, so sectors are fully used); the partial logits are summed
// across warps in shared memory in a fixed order; then one thread per token takes the top-k and threads
// over (token, head) finish dt.
constexpr int kTokTile = 16;
constexpr int kRWarps = 8;
constexpr int kMaxNT = 16;  // up to 128 logits per token

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t ldg32(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const unsigned*>(p)); }

__global__ void __launch_bounds__(kRWarps * 32, 1)
router_mma_kernel(Dims d, int RP, const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ Wr,
                  const __nv_bfloat16* __restrict__ Wdt, const float* __restrict__ bdt, int32_t* __restrict__ idx_out,
                  float* __restrict__ w_out, float* __restrict__ dt_out, int32_t* __restrict__ counts) {
  extern __shared__ __align__(16) float part[];  // [kRWarps][kTokTile][RP + 1] partial logits, then sums
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tok0 = blockIdx.x * kTokTile;
  const int R = d.E + d.H, NT = RP / 8;
  const int g = lane >> 2, c2 = 2 * (lane & 3);
  // this warp's range of 16-wide k-steps
  const int steps = d.D / 16, per = (steps + kRWarps - 1) / kRWarps;
  const int s0 = warp * per, s1 = min(steps, s0 + per);
  const int r0 = min(tok0 + g, d.M - 1), r1 = min(tok0 + g + 8, d.M - 1);  // clamped rows (masked at the end)
  const __nv_bfloat16* xa = X + (size_t)r0 * d.D + c2;
  const __nv_bfloat16* xb = X + (size_t)r1 * d.D + c2;
  const __nv_bfloat16* wrow[kMaxNT];
#pragma unroll
  for (int n = 0; n < kMaxNT; ++n) {
    const int r = min(8 * n + g, R - 1);
    wrow[n] = (r < d.E ? Wr + (size_t)r * d.D : Wdt + (size_t)(r - d.E) * d.D) + c2;
  }
  float acc[kMaxNT][4];
#pragma unroll
  for (int n = 0; n < kMaxNT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll 4
  for (int st = s0; st < s1; ++st) {
    const int k0 = 16 * st;
    const uint32_t a0 = ldg32(xa + k0), a1 = ldg32(xb + k0), a2 = ldg32(xa + k0 + 8), a3 = ldg32(xb + k0 + 8);
#pragma unroll
    for (int n = 0; n < kMaxNT; ++n) {
      if (n < NT) {
        const uint32_t b0 = ldg32(wrow[n] + k0), b1 = ldg32(wrow[n] + k0 + 8);
        mma_bf16_16816(acc[n], a0, a1, a2, a3, b0, b1);
      }
    }
  }
  // partials: c0,c1 at (row g, cols 2c, 2c+1), c2,c3 at (row g + 8, same cols)
  float* mine = part + (size_t)warp * kTokTile * (RP + 1);
#pragma unroll
  for (int n = 0; n < kMaxNT; ++n) {
    if (n < NT) {
      float* p0 = mine + g * (RP + 1) + 8 * n + c2;
      float* p1 = p0 + 8 * (RP + 1);
      p0[0] = acc[n][0]; p0[1] = acc[n][1];
      p1[0] = acc[n][2]; p1[1] = acc[n][3];
    }
  }
  __syncthreads();
  // fixed-order sum over the warps' partials into slot 0
  for (int i = tid; i < kTokTile * RP; i += kRWarps * 32) {
    const int t = i / RP, r = i % RP;
    float v = 0.f;
    for (int w = 0; w < kRWarps; ++w) v += part[(size_t)w * kTokTile * (RP + 1) + t * (RP + 1) + r];
    part[t * (RP + 1) + r] = v;
  }
  __syncthreads();
  // dt for every (token, head)
  for (int i = tid; i < kTokTile * d.H; i += kRWarps * 32) {
    const int t = i / d.H, h = i % d.H, m = tok0 + t;
    if (m < d.M) {
      const float v = part[t * (RP + 1) + d.E + h] + bdt[h];
      const float sp = v > 20.f ? v : log1pf(expf(v));
      dt_out[(size_t)m * d.H + h] = fminf(fmaxf(sp, 1e-3f), 0.1f);
    }
  }
  // top-k, one thread per token: k passes over the E logits, strict '>' so equal values keep the lower index
  if (tid < kTokTile && tok0 + tid < d.M) {
    const int m = tok0 + tid;
    const float* gl = part + tid * (RP + 1);
    unsigned long long taken = 0ull;
    float gsel[8];
    int isel[8];
    for (int j = 0; j < d.k; ++j) {
      int bi = -1;
      float bv = -INFINITY;
      for (int e = 0; e < d.E; ++e) {
        if ((taken >> e) & 1ull) continue;
        if (bi < 0 || gl[e] > bv) { bv = gl[e]; bi = e; }
      }
      taken |= 1ull << bi;
      gsel[j] = bv;
      isel[j] = bi;
    }
    float den = 0.f, ex[8];
    for (int j = 0; j < d.k; ++j) { ex[j] = expf(gsel[j] - gsel[0]); den += ex[j]; }
    for (int j = 0; j < d.k; ++j) {
      idx_out[(size_t)m * d.k + j] = isel[j];
      w_out[(size_t)m * d.k + j] = ex[j] / den;
      if (counts) atomicAdd(&counts[(size_t)((m * d.k + j) / kDispatchTile) * d.E + isel[j]], 1);
    }
  }
}
}  // namespace

cudaError_t launch_router(const Dims& d, const void* X, const swimba_weights& w, int32_t* idx, float* wts,
                          float* dt, int32_t* counts, cudaStream_t s) {
  const int R = d.E + d.H;
  if (d.dtype == SWIMBA_BF16 && R <= 8 * kMaxNT) {
    const int RP = (R + 7) / 8 * 8;
    const size_t smem = (size_t)kRWarps * kTokTile * (RP + 1) * 4;
    cudaError_t e = cudaFuncSetAttribute(router_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    router_mma_kernel<<<ceil_div(d.M, kTokTile), kRWarps * 32, smem, s>>>(d, RP, (const __nv_bfloat16*)X,
                                                                         (const __nv_bfloat16*)w.w_router,
                                                                         (const __nv_bfloat16*)w.w_dt, w.b_dt, idx,
                                                                         wts, dt, counts);
  } else {
    const size_t smem = sizeof(float) * (size_t)kRouterWarps * (d.D + R);
    if (d.dtype == SWIMBA_BF16) {
      auto k = router_simt_kernel<__nv_bfloat16>;
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      k<<<ceil_div(d.M, kRouterWarps), kRouterWarps * 32, smem, s>>>(
          d, (const __nv_bfloat16*)X, (const __nv_bfloat16*)w.w_router, (const __nv_bfloat16*)w.w_dt, w.b_dt, idx,
          wts, dt, counts);
    } else {
      auto k = router_simt_kernel<float>;
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      k<<<ceil_div(d.M, kRouterWarps), kRouterWarps * 32, smem, s>>>(d, (const float*)X, (const float*)w.w_router,
                                                                      (const float*)w.w_dt, w.b_dt, idx, wts, dt,
                                                                      counts);
    }
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swimba
