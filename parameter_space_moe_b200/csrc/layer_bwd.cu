// Gradients of the whole layer: the stages after the scan gradients, in fp32.
//
// Paper: Swimba notes, Method flowchart (router -> expert projections -> parameter-space mixing -> one
// recurrence) differentiated stage by stage in reverse; the notes train the model (loss function / training
// strategy).  With the scan's gradients (dBpi, dXs, dC~, d dt) in hand:
//   mix     dz_j = [dXs_j | pi_j dBpi_j | pi_j dC~]  per (token, slot);  dpi_j = <B_j, dBpi_j> + <C_j, dC~>
//   router  dg_j = pi_j (dpi_j - sum_i pi_i dpi_i) on the active set (held fixed: a top-k choice has no
//           gradient);  du = d dt * sigmoid(u) where the clamp of dt = clamp(softplus(u)) is not active,
//           with sigmoid(u) = 1 - e^{-softplus(u)} = -expm1(-dt)
//   linear  dW_exp[e] = sum over the (token, slot) rows of expert e of dz (x) X_token
//           dX_t = sum_j W_exp[K_tj]^T dz_tj + W_r^T dg_t + W_dt^T du_t;  dW_r = dg^T X;  dW_dt = du^T X;
//           db_dt = sum_t du_t.
// The (token, slot) rows are visited in the dispatch's expert order (perm, offsets, row tiles), as in the
// forward projection.  The two expert products run on the tensor cores for bf16 layers (grad_tc.cu, on a
// bf16 hi/lo split of dz) and on the CUDA-core kernels below for fp32 layers.
#include "common.cuh"

namespace swimba {

namespace {
constexpr int kT = 64;   // output tile edge of the CUDA-core GEMMs
constexpr int kK = 16;   // contraction step

// mix: one CTA per (token, slot) pair p.  fp32 layers: z (raw projection) is overwritten by dz.  bf16 layers
// (kSplit): dz goes straight into the pair's padded row of the tensor-core products' operand as a bf16 split,
// hi = bf16(dz) in columns [0, W_e), lo = bf16(dz - hi) in [Wp, Wp + W_e), zeros up to each half's end.
template <bool kSplit>
__global__ void __launch_bounds__(256) mix_bwd_kernel(Dims d, float* __restrict__ z, const float* __restrict__ wts,
                                                      const float* __restrict__ dbpi, const float* __restrict__ dxs,
                                                      const float* __restrict__ dct, float* __restrict__ dpi,
                                                      const int32_t* __restrict__ rp_of_p,
                                                      __nv_bfloat16* __restrict__ dzs, int Wp) {
  __shared__ float red[8];
  const size_t p = blockIdx.x;
  const size_t m = p / d.k;
  const float pi = wts[p];
  float* zr = z + p * d.We;
  const float* gb = dbpi + p * d.GN;
  const float* gc = dct + m * d.GN;
  float part = 0.f;
  for (int c = threadIdx.x; c < d.GN; c += blockDim.x)
    part = fmaf(zr[d.HP + c], gb[c], fmaf(zr[d.HP + d.GN + c], gc[c], part));
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
  __syncthreads();  // every read of z is done before it is overwritten below
  if (threadIdx.x == 0) {
    float v = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v += red[w];
    dpi[p] = v;
  }
  const float* gx = dxs + p * d.HP;
  if constexpr (kSplit) {
    // pairs of columns (H*P and G*N are even, so a pair never straddles two streams)
    __nv_bfloat162* hi = reinterpret_cast<__nv_bfloat162*>(dzs + (size_t)rp_of_p[p] * 2 * Wp);
    __nv_bfloat162* lo = hi + Wp / 2;
    for (int c2 = threadIdx.x; c2 < Wp / 2; c2 += blockDim.x) {
      const int c = 2 * c2;
      float2 v = make_float2(0.f, 0.f);
      if (c < d.HP) v = make_float2(gx[c], gx[c + 1]);
      else if (c < d.HP + d.GN) v = make_float2(pi * gb[c - d.HP], pi * gb[c - d.HP + 1]);
      else if (c < d.We) v = make_float2(pi * gc[c - d.HP - d.GN], pi * gc[c - d.HP - d.GN + 1]);
      const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
      const float2 hf = __bfloat1622float2(h);
      hi[c2] = h;
      lo[c2] = __floats2bfloat162_rn(v.x - hf.x, v.y - hf.y);
    }
  } else {
    for (int c = threadIdx.x; c < d.HP; c += blockDim.x) zr[c] = gx[c];
    for (int c = threadIdx.x; c < d.GN; c += blockDim.x) {
      zr[d.HP + c] = pi * gb[c];
      zr[d.HP + d.GN + c] = pi * gc[c];
    }
  }
}

// router and dt: dg [M][E] (zero off the active set), du [M][H]
__global__ void router_bwd_kernel(Dims d, const int32_t* __restrict__ idx, const float* __restrict__ wts,
                                  const float* __restrict__ dpi, const float* __restrict__ dt,
                                  const float* __restrict__ ddt, float* __restrict__ dg, float* __restrict__ du) {
  const size_t m = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (m >= (size_t)d.M) return;
  float s = 0.f;
  for (int j = 0; j < d.k; ++j) s = fmaf(wts[m * d.k + j], dpi[m * d.k + j], s);
  for (int e = 0; e < d.E; ++e) dg[m * d.E + e] = 0.f;
  for (int j = 0; j < d.k; ++j) {
    const int e = idx[m * d.k + j];
    if (e >= 0 && e < d.E) dg[m * d.E + e] = wts[m * d.k + j] * (dpi[m * d.k + j] - s);
  }
  for (int h = 0; h < d.H; ++h) {
    const float v = dt[m * d.H + h];
    du[m * d.H + h] = (v > 1e-3f && v < 0.1f) ? ddt[m * d.H + h] * -expm1f(-v) : 0.f;
  }
}

// 128 x 128 output tiles, 8 x 8 per thread (rows ty * 8 .., columns tx * 8 ..), contraction staged 8 at a
// time through two shared-memory buffers: each thread loads the next stage's four A and four B values into
// registers (one 16-byte dz load, one 4-element operand load) while the current stage is multiplied, so one
// barrier per stage suffices and the global latency hides behind 512 FMAs.  W_e % 16 == 0 and D % 8 == 0,
// so a 4-wide group never straddles a matrix edge.
constexpr int kBT2 = 128, kBK2 = 8, kLd2 = kBT2 + 4;
struct Stage {
  float A[kBK2][kLd2];
  float B[kBK2][kLd2];
};

__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__device__ __forceinline__ void mac8x8(const Stage& S, int ty, int tx, float (&acc)[8][8]) {
#pragma unroll
  for (int kk = 0; kk < kBK2; ++kk) {
    const float4 a0 = *reinterpret_cast<const float4*>(&S.A[kk][ty * 8]);
    const float4 a1 = *reinterpret_cast<const float4*>(&S.A[kk][ty * 8 + 4]);
    const float4 b0 = *reinterpret_cast<const float4*>(&S.B[kk][tx * 8]);
    const float4 b1 = *reinterpret_cast<const float4*>(&S.B[kk][tx * 8 + 4]);
    const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
}

// dXp[p][n] = sum_c dz[p][c] W_exp[e][c][n] for the rows of one 128-row dispatch tile (expert e), 128 columns n.
// A stage: A = dz[rows][c0 .. c0+8) transposed (thread: row tid/2, columns 4 (tid&1) ..), B = W_e[c0 .. c0+8)[n]
// (thread: row tid/32, columns 4 (tid&31) ..).
template <class T>
__global__ void __launch_bounds__(256, 2)
dx_experts_kernel(Dims d, const float* __restrict__ dz, const T* __restrict__ W, const int32_t* __restrict__ perm,
                  const int32_t* __restrict__ tiles, const int32_t* __restrict__ ntiles,
                  const int32_t* __restrict__ offsets, float* __restrict__ dxp) {
  __shared__ __align__(16) Stage st[2];
  __shared__ int pr[kRowTile];
  if ((int)blockIdx.x >= *ntiles) return;
  const int e = tiles[2 * blockIdx.x], row0 = tiles[2 * blockIdx.x + 1];
  const int rows = min(kRowTile, offsets[e + 1] - row0);
  const int n0 = blockIdx.y * kBT2;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  for (int r = tid; r < kRowTile; r += 256) pr[r] = r < rows ? perm[row0 + r] : -1;
  __syncthreads();
  const T* We = W + (size_t)e * d.We * d.D;
  const int ar = tid >> 1, ak = (tid & 1) * 4, bk = tid >> 5, bn = (tid & 31) * 4;
  const int ap = pr[ar];
  const float* arow = dz + (size_t)max(ap, 0) * d.We + ak;
  const T* bptr = We + (size_t)bk * d.D + n0 + bn;
  const bool aok = ap >= 0, bok = n0 + bn < d.D;
  const size_t bstep = (size_t)kBK2 * d.D;
  const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
  auto fetch = [&](int c0, float4& a, float4& b) {
    a = (aok && c0 + ak < d.We) ? load4(arow + c0) : z4;
    b = (bok && c0 + bk < d.We) ? load4(bptr) : z4;
    bptr += bstep;
  };
  float4 a, b;
  fetch(0, a, b);
  float acc[8][8] = {};
  int buf = 0;
  for (int c0 = 0; c0 < d.We; c0 += kBK2) {
    Stage& S = st[buf];
    S.A[ak][ar] = a.x; S.A[ak + 1][ar] = a.y; S.A[ak + 2][ar] = a.z; S.A[ak + 3][ar] = a.w;
    *reinterpret_cast<float4*>(&S.B[bk][bn]) = b;
    __syncthreads();
    if (c0 + kBK2 < d.We) fetch(c0 + kBK2, a, b);
    mac8x8(S, ty, tx, acc);
    buf ^= 1;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = ty * 8 + i;
    if (r >= rows) continue;
    const int p = pr[r];
#pragma unroll
    for (int j = 0; j < 8; j += 4) {
      const int n = n0 + tx * 8 + j;
      if (n < d.D)
        *reinterpret_cast<float4*>(dxp + (size_t)p * d.D + n) =
            make_float4(acc[i][j], acc[i][j + 1], acc[i][j + 2], acc[i][j + 3]);
    }
  }
}

// dW_exp[e][c][n] = sum over all of expert e's (token, slot) rows of dz[p][c] X[token(p)][n]: one CTA per
// (expert, 128 W_e columns c, 128 D columns n) walks the expert's sorted rows 8 at a time (plain stores, no
// atomics).  A stage: A = dz[row][c0 ..], B = X[token][n0 ..] (thread: row tid/32, columns 4 (tid&31) ..).
template <class T>
__global__ void __launch_bounds__(256, 2)
dw_experts_kernel(Dims d, const float* __restrict__ dz, const T* __restrict__ X, const int32_t* __restrict__ perm,
                  const int32_t* __restrict__ offsets, float* __restrict__ dW) {
  __shared__ __align__(16) Stage st[2];
  const int e = blockIdx.x, c0 = blockIdx.y * kBT2, n0 = blockIdx.z * kBT2;
  const int rb = offsets[e], re = offsets[e + 1];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int kr = tid >> 5, kc = (tid & 31) * 4;
  const bool aok = c0 + kc < d.We, bok = n0 + kc < d.D;
  const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
  auto fetch = [&](int r0, float4& a, float4& b) {
    const int p = r0 + kr < re ? perm[r0 + kr] : -1;
    a = (p >= 0 && aok) ? load4(dz + (size_t)p * d.We + c0 + kc) : z4;
    b = (p >= 0 && bok) ? load4(X + (size_t)(p / d.k) * d.D + n0 + kc) : z4;
  };
  float4 a, b;
  if (rb < re) fetch(rb, a, b);
  float acc[8][8] = {};
  int buf = 0;
  for (int r0 = rb; r0 < re; r0 += kBK2) {
    Stage& S = st[buf];
    *reinterpret_cast<float4*>(&S.A[kr][kc]) = a;
    *reinterpret_cast<float4*>(&S.B[kr][kc]) = b;
    __syncthreads();
    if (r0 + kBK2 < re) fetch(r0 + kBK2, a, b);
    mac8x8(S, ty, tx, acc);
    buf ^= 1;
  }
  float* out = dW + (size_t)e * d.We * d.D;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = c0 + ty * 8 + i;
    if (c >= d.We) continue;
#pragma unroll
    for (int j = 0; j < 8; j += 4) {
      const int n = n0 + tx * 8 + j;
      if (n < d.D)
        *reinterpret_cast<float4*>(out + (size_t)c * d.D + n) =
            make_float4(acc[i][j], acc[i][j + 1], acc[i][j + 2], acc[i][j + 3]);
    }
  }
}

// out[r][n] += sum over a 256-token slice of G[m][r] X[m][n] (dW_r from dg, dW_dt from du); 64-row tiles of r
template <class T>
__global__ void __launch_bounds__(256)
dw_dense_kernel(int M, int R, int D, const float* __restrict__ G, const T* __restrict__ X, float* __restrict__ out) {
  __shared__ float As[kK][kT + 4];
  __shared__ float Bs[kK][kT + 4];
  const int n0 = blockIdx.x * kT, m_begin = blockIdx.y * 256, m_end = min(M, m_begin + 256), r0 = blockIdx.z * kT;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float acc[4][4] = {};
  for (int m0 = m_begin; m0 < m_end; m0 += kK) {
    for (int i = tid; i < kK * kT; i += 256) {
      const int kk = i / kT, c = i % kT, m = m0 + kk;
      As[kk][c] = (m < m_end && r0 + c < R) ? G[(size_t)m * R + r0 + c] : 0.f;
      Bs[kk][c] = (m < m_end && n0 + c < D) ? to_f32(X[(size_t)m * D + n0 + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + ty + 16 * i;
    if (r >= R) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n < D) atomicAdd(&out[(size_t)r * D + n], acc[i][j]);
    }
  }
}

// dX[m][n] = sum_j dXp[m k + j][n] + sum_e dg[m][e] W_r[e][n] + sum_h du[m][h] W_dt[h][n];  db_dt[h] += du
template <class T>
__global__ void dx_final_kernel(Dims d, const float* __restrict__ dxp, const float* __restrict__ dg,
                                const float* __restrict__ du, const T* __restrict__ Wr, const T* __restrict__ Wdt,
                                float* __restrict__ dX) {
  const size_t total = (size_t)d.M * d.D;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const size_t m = i / d.D;
    const int n = (int)(i % d.D);
    float v = 0.f;
    for (int j = 0; j < d.k; ++j) v += dxp[(m * d.k + j) * d.D + n];
    for (int e = 0; e < d.E; ++e) v = fmaf(dg[m * d.E + e], to_f32(Wr[(size_t)e * d.D + n]), v);
    for (int h = 0; h < d.H; ++h) v = fmaf(du[m * d.H + h], to_f32(Wdt[(size_t)h * d.D + n]), v);
    dX[i] = v;
  }
}

__global__ void db_kernel(Dims d, const float* __restrict__ du, float* __restrict__ db) {
  const int h = blockIdx.x;
  float s = 0.f;
  for (int m = threadIdx.x; m < d.M; m += blockDim.x) s += du[(size_t)m * d.H + h];
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v += red[w];
    db[h] = v;
  }
}

// 1. the mix and router gradients: dz (over z, or as the bf16 split of the tensor-core products), dpi, dg, du
cudaError_t launch_mix_router(const Dims& d, const LayerBwdPtrs& q, cudaStream_t s) {
  if (d.dtype == SWIMBA_BF16) {
    const cudaError_t e = launch_grad_tc_pack(d, q.xsorted, q.perm, q.offsets, q.poff, q.prow, q.rp_of_p, q.dzs,
                                              q.xsp, s);
    if (e != cudaSuccess) return e;
    mix_bwd_kernel<true><<<d.M * d.k, 256, 0, s>>>(d, q.z, q.wts, q.dbpi, q.dxs, q.dct, q.dpi, q.rp_of_p,
                                                   (__nv_bfloat16*)q.dzs, grad_tc_wp(d));
  } else {
    mix_bwd_kernel<false><<<d.M * d.k, 256, 0, s>>>(d, q.z, q.wts, q.dbpi, q.dxs, q.dct, q.dpi, nullptr, nullptr, 0);
  }
  router_bwd_kernel<<<ceil_div(d.M, 128), 128, 0, s>>>(d, q.idx, q.wts, q.dpi, q.dt, q.ddt, q.dg, q.du);
  count_launches(2);
  return cudaGetLastError();
}

// 2. the expert products dXp = dz W_e and dW_exp = dz^T X
template <class T>
cudaError_t launch_experts_typed(const Dims& d, const LayerBwdPtrs& q, cudaStream_t s) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    // tensor cores on the bf16 hi/lo split of dz (laid out by the mix gradient)
    return launch_grad_tc(d, q.w_exp, q.offsets, q.poff, q.prow, q.dzs, q.xsp, q.dxp, q.dW_exp, q.st, s);
  } else {
    const dim3 gx(max_row_tiles(d), ceil_div(d.D, kBT2));
    dx_experts_kernel<T><<<gx, 256, 0, s>>>(d, q.z, (const T*)q.w_exp, q.perm, q.tiles, q.ntiles, q.offsets, q.dxp);
    const dim3 gw(d.E, ceil_div(d.We, kBT2), ceil_div(d.D, kBT2));
    dw_experts_kernel<T><<<gw, 256, 0, s>>>(d, q.z, (const T*)q.X, q.perm, q.offsets, q.dW_exp);
    count_launches(2);
    return cudaGetLastError();
  }
}

// 3. the router and dt weight gradients, db_dt, and dX summed over the slots with the router and dt terms
template <class T>
cudaError_t launch_linear_typed(const Dims& d, const LayerBwdPtrs& q, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(q.dW_r, 0, (size_t)d.E * d.D * 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(q.dW_dt, 0, (size_t)d.H * d.D * 4, s);
  if (e != cudaSuccess) return e;
  dw_dense_kernel<T><<<dim3(ceil_div(d.D, kT), ceil_div(d.M, 256), ceil_div(d.E, kT)), 256, 0, s>>>(
      d.M, d.E, d.D, q.dg, (const T*)q.X, q.dW_r);
  dw_dense_kernel<T><<<dim3(ceil_div(d.D, kT), ceil_div(d.M, 256), ceil_div(d.H, kT)), 256, 0, s>>>(
      d.M, d.H, d.D, q.du, (const T*)q.X, q.dW_dt);
  db_kernel<<<d.H, 256, 0, s>>>(d, q.du, q.db_dt);
  dx_final_kernel<T><<<148 * 8, 256, 0, s>>>(d, q.dxp, q.dg, q.du, (const T*)q.w_r, (const T*)q.w_dt, q.dX);
  count_launches(4);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_layer_bwd_tail(const Dims& d, const LayerBwdPtrs& q, int part, cudaStream_t s) {
  const bool bf = d.dtype == SWIMBA_BF16;
  switch (part) {
    case 0: return launch_mix_router(d, q, s);
    case 1: return bf ? launch_experts_typed<__nv_bfloat16>(d, q, s) : launch_experts_typed<float>(d, q, s);
    case 2: return bf ? launch_linear_typed<__nv_bfloat16>(d, q, s) : launch_linear_typed<float>(d, q, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace swimba
