// Router and dt projection.
//
// Paper: Swimba notes, Method, flowchart node "token router R(X_t)" and key design 1
// (pi_t = softmax(g_t) over the active set K_t).  Per token t:
//   g_t,e  = W_r[e] . X_t                         (fp32 accumulation)
//   K_t    = the k largest g_t,e, largest first, equal values -> lower e
//   pi_t,j = exp(g_{K_j} - g_{K_0}) / sum_j' exp(g_{K_j'} - g_{K_0})
//   dt_t,h = clamp(softplus(W_dt[h] . X_t + b_dt[h]), 1e-3, 0.1)
// The E + H dot products per token form a skinny GEMM [M x D] x [D x (E + H)].  bf16 layers run it on
// the tcgen05 kernel in router_tc.cu where its logit row fits; otherwise on the warp-level tensor-core
// path here (mma.sync m16n8k16, fp32 accumulate): a CTA of 4 warps owns 64 tokens and streams X and the
// stacked [W_r; W_dt] through padded shared memory in 64-wide K chunks (cp.async, 4-stage pipeline);
// then threads over (token, head) finish dt and one thread per token takes the top-k.  The fp32 layer
// keeps a CUDA-core kernel (one warp per token, fixed xor butterfly reductions).
#include "common.cuh"

namespace swimba {

namespace {

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
constexpr int kMT = 64;           // tokens per CTA
constexpr int kKC = 64;           // K chunk
constexpr int kLd = kKC + 8;      // padded shared row (144 B: conflict-free ldmatrix)
constexpr int kMaxNT = 16;        // up to 128 logits per token
constexpr int kStagesR = 4;       // cp.async pipeline depth

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(dst);
  const int n = valid ? 16 : 0;  // zero-fill when invalid
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(128)
router_mma_kernel(Dims d, int RP, const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ Wr,
                  const __nv_bfloat16* __restrict__ Wdt, const float* __restrict__ bdt, int32_t* __restrict__ idx_out,
                  float* __restrict__ w_out, float* __restrict__ dt_out, int32_t* __restrict__ counts) {
  extern __shared__ __align__(16) uint8_t rsm[];
  __nv_bfloat16* Xs = reinterpret_cast<__nv_bfloat16*>(rsm);   // [stages][kMT][kLd]
  __nv_bfloat16* Ws = Xs + kStagesR * kMT * kLd;                 // [stages][RP][kLd]
  float* G = reinterpret_cast<float*>(Ws + kStagesR * RP * kLd); // [kMT][RP + 1]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tok0 = blockIdx.x * kMT;
  const int R = d.E + d.H, NT = RP / 8, nkc = d.D / kKC;

  auto load = [&](int stage, int kc) {
    if (kc < nkc) {
      const int k0 = kc * kKC;
      __nv_bfloat16* xs = Xs + stage * kMT * kLd;
      __nv_bfloat16* ws = Ws + stage * RP * kLd;
      for (int i = tid; i < kMT * (kKC / 8); i += 128) {
        const int r = i >> 3, c = i & 7;
        const bool v = tok0 + r < d.M;
        cp_async16(xs + r * kLd + 8 * c, X + (size_t)(v ? tok0 + r : 0) * d.D + k0 + 8 * c, v);
      }
      for (int i = tid; i < RP * (kKC / 8); i += 128) {
        const int r = i >> 3, c = i & 7;
        const __nv_bfloat16* src = r < d.E ? Wr + (size_t)r * d.D : Wdt + (size_t)(r < R ? r - d.E : 0) * d.D;
        cp_async16(ws + r * kLd + 8 * c, src + k0 + 8 * c, r < R);
      }
    }
    cp_async_commit();  // an empty group past the end keeps the group count uniform
  };

  float acc[kMaxNT][4];
#pragma unroll
  for (int n = 0; n < kMaxNT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

#pragma unroll
  for (int st = 0; st < kStagesR - 1; ++st) load(st, st);
  for (int kc = 0; kc < nkc; ++kc) {
    const int stage = kc % kStagesR;
    cp_async_wait<kStagesR - 2>();
    __syncthreads();
    load((kc + kStagesR - 1) % kStagesR, kc + kStagesR - 1);  // refills the stage read in iteration kc - 1
    const uint32_t xb = (uint32_t)__cvta_generic_to_shared(Xs + stage * kMT * kLd);
    const uint32_t wb = (uint32_t)__cvta_generic_to_shared(Ws + stage * RP * kLd);
#pragma unroll
    for (int ks = 0; ks < kKC / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(xb + (uint32_t)(((16 * warp + (lane & 15)) * kLd + 16 * ks + (lane >> 4) * 8) * 2), a0, a1, a2, a3);
#pragma unroll
      for (int np = 0; np < kMaxNT / 2; ++np) {
        if (2 * np < NT) {
          uint32_t b0, b1, b2, b3;
          const int n = 16 * np + (lane & 7) + 8 * (lane >> 4);
          ldmatrix_x4(wb + (uint32_t)((n * kLd + 16 * ks + ((lane >> 3) & 1) * 8) * 2), b0, b1, b2, b3);
          mma_bf16_16816(acc[2 * np], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  // logits -> shared memory: c0,c1 at (row g, cols 2c, 2c+1), c2,c3 at (row g + 8, same cols)
  const int gr = lane >> 2, gc = 2 * (lane & 3);
#pragma unroll
  for (int n = 0; n < kMaxNT; ++n) {
    if (n < NT) {
      float* r0 = G + (16 * warp + gr) * (RP + 1) + 8 * n + gc;
      float* r1 = r0 + 8 * (RP + 1);
      r0[0] = acc[n][0]; r0[1] = acc[n][1];
      r1[0] = acc[n][2]; r1[1] = acc[n][3];
    }
  }
  __syncthreads();
  // dt for every (token, head), then the top-k with one thread per token: k passes over the E logits,
  // strict '>' so equal values keep the lower index
  for (int i = tid; i < kMT * d.H; i += 128) {
    const int t = i / d.H, h = i % d.H, m = tok0 + t;
    if (m < d.M) {
      const float v = G[t * (RP + 1) + d.E + h] + bdt[h];
      const float sp = v > 20.f ? v : log1pf(expf(v));
      dt_out[(size_t)m * d.H + h] = fminf(fmaxf(sp, 1e-3f), 0.1f);
    }
  }
  if (tid < kMT && tok0 + tid < d.M) {
    const int m = tok0 + tid;
    const float* gl = G + tid * (RP + 1);
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
                          float* dt, int32_t* counts, unsigned* st, cudaStream_t s, bool after_zero) {
  const int R = d.E + d.H;
  if (st && router_tc_supported(d)) {
    const cudaError_t e = launch_router_tc(d, X, w, idx, wts, dt, counts, st, s, after_zero);
    if (e != cudaErrorNotSupported) return e;
  }
  if (d.dtype == SWIMBA_BF16 && R <= 8 * kMaxNT) {
    const int RP = (R + 15) / 16 * 16;
    const size_t smem = (size_t)kStagesR * (kMT + RP) * kLd * 2 + (size_t)kMT * (RP + 1) * 4;
    cudaError_t e = set_max_dynamic_smem((const void*)router_mma_kernel, smem);
    if (e != cudaSuccess) return e;
    router_mma_kernel<<<ceil_div(d.M, kMT), 128, smem, s>>>(d, RP, (const __nv_bfloat16*)X,
                                                             (const __nv_bfloat16*)w.w_router,
                                                             (const __nv_bfloat16*)w.w_dt, w.b_dt, idx, wts, dt,
                                                             counts);
  } else {
    const size_t smem = sizeof(float) * (size_t)kRouterWarps * (d.D + R);
    if (d.dtype == SWIMBA_BF16) {
      auto k = router_simt_kernel<__nv_bfloat16>;
      cudaError_t e = set_max_dynamic_smem((const void*)k, smem);
      if (e != cudaSuccess) return e;
      k<<<ceil_div(d.M, kRouterWarps), kRouterWarps * 32, smem, s>>>(
          d, (const __nv_bfloat16*)X, (const __nv_bfloat16*)w.w_router, (const __nv_bfloat16*)w.w_dt, w.b_dt, idx,
          wts, dt, counts);
    } else {
      auto k = router_simt_kernel<float>;
      cudaError_t e = set_max_dynamic_smem((const void*)k, smem);
      if (e != cudaSuccess) return e;
      k<<<ceil_div(d.M, kRouterWarps), kRouterWarps * 32, smem, s>>>(d, (const float*)X, (const float*)w.w_router,
                                                                      (const float*)w.w_dt, w.b_dt, idx, wts, dt,
                                                                      counts);
    }
  }
  count_launches(1);
  return cudaGetLastError();
}

namespace {
__global__ void zero_u32_kernel(unsigned* p, size_t n) {
  griddep_launch_dependents();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) p[i] = 0u;
}
}  // namespace

cudaError_t launch_zero_u32(unsigned* p, size_t n, cudaStream_t s) {
  const size_t blocks = (n + 255) / 256;
  zero_u32_kernel<<<(unsigned)(blocks < 148 ? (blocks > 0 ? blocks : 1) : 148), 256, 0, s>>>(p, n);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swimba
