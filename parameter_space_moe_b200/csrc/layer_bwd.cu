// Gradients of the whole layer: the stages after the scan gradients, fp32 values and accumulation.
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

// mix: one CTA per (token, slot) pair p.  fp32 layers: z (raw projection) is overwritten by dz.  bf16 layers
// (kSplit): dz goes straight into the pair's padded row of the tensor-core products' operand as a bf16 split,
// hi = bf16(dz) in columns [0, W_e), lo = bf16(dz - hi) in [Wp, Wp + W_e), zeros up to each half's end.
template <bool kSplit>
__global__ void __launch_bounds__(256) mix_bwd_kernel(Dims d, float* __restrict__ z, const float* __restrict__ wts,
                                                      const float* __restrict__ dbpi, const float* __restrict__ dxs,
                                                      const float* __restrict__ dct, float* __restrict__ dpi,
                                                      const int32_t* __restrict__ rp_of_p,
                                                      __nv_bfloat16* __restrict__ dzs, int Wp) {
  // 16-byte vectors throughout: H*P and G*N are multiples of 16, so a 4-column group never straddles streams
  __shared__ float red[8];
  const size_t p = blockIdx.x;
  const size_t m = p / d.k;
  const float pi = wts[p];
  float* zr = z + p * d.We;
  const float4* zb = reinterpret_cast<const float4*>(zr + d.HP);
  const float4* zc = reinterpret_cast<const float4*>(zr + d.HP + d.GN);
  const float4* gb = reinterpret_cast<const float4*>(dbpi + p * d.GN);
  const float4* gc = reinterpret_cast<const float4*>(dct + m * d.GN);
  const int GN4 = d.GN / 4;
  float part = 0.f;
#pragma unroll 4
  for (int c = threadIdx.x; c < GN4; c += blockDim.x) {
    const float4 b = zb[c], g = gb[c], cc = zc[c], h = gc[c];
    part = fmaf(b.x, g.x, fmaf(b.y, g.y, fmaf(b.z, g.z, fmaf(b.w, g.w, part))));
    part = fmaf(cc.x, h.x, fmaf(cc.y, h.y, fmaf(cc.z, h.z, fmaf(cc.w, h.w, part))));
  }
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
  __syncthreads();  // every read of z is done before it is overwritten below
  if (threadIdx.x == 0) {
    float v = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v += red[w];
    dpi[p] = v;
  }
  const float4* gx = reinterpret_cast<const float4*>(dxs + p * d.HP);
  const int HP4 = d.HP / 4, We4 = d.We / 4;
  // column group c4 of dz = [dXs | pi dBpi | pi dC~]
  auto dz4 = [&](int c4) {
    if (c4 < HP4) return gx[c4];
    float4 v = c4 < HP4 + GN4 ? gb[c4 - HP4] : gc[c4 - HP4 - GN4];
    v.x *= pi; v.y *= pi; v.z *= pi; v.w *= pi;
    return v;
  };
  if constexpr (kSplit) {
    uint2* hi = reinterpret_cast<uint2*>(dzs + (size_t)rp_of_p[p] * 2 * Wp);
    uint2* lo = hi + Wp / 4;
#pragma unroll 4
    for (int c4 = threadIdx.x; c4 < Wp / 4; c4 += blockDim.x) {
      const float4 v = c4 < We4 ? dz4(c4) : make_float4(0.f, 0.f, 0.f, 0.f);
      const __nv_bfloat162 h0 = __floats2bfloat162_rn(v.x, v.y), h1 = __floats2bfloat162_rn(v.z, v.w);
      const float2 f0 = __bfloat1622float2(h0), f1 = __bfloat1622float2(h1);
      const __nv_bfloat162 l0 = __floats2bfloat162_rn(v.x - f0.x, v.y - f0.y);
      const __nv_bfloat162 l1 = __floats2bfloat162_rn(v.z - f1.x, v.w - f1.y);
      hi[c4] = make_uint2(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
      lo[c4] = make_uint2(*reinterpret_cast<const uint32_t*>(&l0), *reinterpret_cast<const uint32_t*>(&l1));
    }
  } else {
    float4* zw = reinterpret_cast<float4*>(zr);
#pragma unroll 4
    for (int c4 = threadIdx.x; c4 < We4; c4 += blockDim.x) zw[c4] = dz4(c4);
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

// The gate rows r < E + H of a token: dg[m][r] for r < E, then du[m][r - E].
__device__ __forceinline__ float gate_at(const Dims& d, const float* __restrict__ dg, const float* __restrict__ du,
                                         int m, int r) {
  return r < d.E ? dg[(size_t)m * d.E + r] : du[(size_t)m * d.H + (r - d.E)];
}

// dW_r[e][n] = sum_m dg[m][e] X[m][n] and dW_dt[h][n] = sum_m du[m][h] X[m][n] as one product over the gate
// rows: a CTA takes 32 gate rows x 128 columns over a 128-token slice, 16 tokens per stage through two
// shared-memory buffers (each thread fetches the next stage's 8 X values in one 16-byte load and 2 gate values
// while the current stage is multiplied); thread (column c, row half) keeps 16 accumulators; atomic adds into
// the zeroed outputs.  D % 8 == 0, so an 8-column group never straddles the matrix edge.
constexpr int kGR = 32, kGC = 128, kGM = 128, kGK = 16;
__device__ __forceinline__ void load8(const float* p, float (&f)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __bfloat1622float2(h[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}

template <class T>
__global__ void __launch_bounds__(256)
dw_gate_kernel(Dims d, const float* __restrict__ dg, const float* __restrict__ du, const T* __restrict__ X,
               float* __restrict__ dWr, float* __restrict__ dWdt) {
  __shared__ __align__(16) float Gs[2][kGK][kGR];
  __shared__ __align__(16) float Xs[2][kGK][kGC];
  const int R = d.E + d.H;
  const int n0 = blockIdx.x * kGC, m_begin = blockIdx.y * kGM, m_end = min(d.M, m_begin + kGM);
  const int r0 = blockIdx.z * kGR;
  const int tid = threadIdx.x, c = tid & (kGC - 1), rh = tid >> 7;  // a warp shares its row half
  const int xr = tid >> 4, xc = (tid & 15) * 8;                      // X stage: token xr, columns xc ..
  float xv[8], gv[2];
  auto fetch = [&](int m0) {
    const int m = m0 + xr;
    if (m < m_end && n0 + xc < d.D) {
      load8(X + (size_t)m * d.D + n0 + xc, xv);
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) xv[u] = 0.f;
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = 2 * tid + u, mm = m0 + i / kGR, r = r0 + i % kGR;
      gv[u] = (mm < m_end && r < R) ? gate_at(d, dg, du, mm, r) : 0.f;
    }
  };
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  fetch(m_begin);
  int buf = 0;
  for (int m0 = m_begin; m0 < m_end; m0 += kGK) {
#pragma unroll
    for (int u = 0; u < 8; ++u) Xs[buf][xr][xc + u] = xv[u];
#pragma unroll
    for (int u = 0; u < 2; ++u) (&Gs[buf][0][0])[2 * tid + u] = gv[u];
    __syncthreads();
    if (m0 + kGK < m_end) fetch(m0 + kGK);
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
      const float x = Xs[buf][kk][c];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = fmaf(Gs[buf][kk][rh * 16 + i], x, acc[i]);
    }
    buf ^= 1;
  }
  const int n = n0 + c;
  if (n >= d.D) return;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = r0 + rh * 16 + i;
    if (r < d.E) atomicAdd(&dWr[(size_t)r * d.D + n], acc[i]);
    else if (r < R) atomicAdd(&dWdt[(size_t)(r - d.E) * d.D + n], acc[i]);
  }
}

// dX[m][n] = sum_j dXp[m k + j][n] + sum_{r < E + H} gate[m][r] Wg[r][n]  (Wg = W_r rows, then W_dt rows):
// 128 x 128 output tiles on the 8 x 8-per-thread tile code of the expert products, K = E + H staged 8 at a
// time; each thread starts from its outputs' slot sums (16-byte loads, all issued before the first stage).
template <class T>
__global__ void __launch_bounds__(256, 2)
dx_final_kernel(Dims d, const float* __restrict__ dxp, const float* __restrict__ dg, const float* __restrict__ du,
                const T* __restrict__ Wr, const T* __restrict__ Wdt, float* __restrict__ dX) {
  __shared__ __align__(16) Stage st;
  const int R = d.E + d.H;
  const int n0 = blockIdx.x * kBT2, m0 = blockIdx.y * kBT2;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + ty * 8 + i;
#pragma unroll
    for (int jv = 0; jv < 8; jv += 4) {
      const int n = n0 + tx * 8 + jv;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (m < d.M && n < d.D) {
        const float* row = dxp + (size_t)m * d.k * d.D + n;
#pragma unroll
        for (int j = 0; j < 8; ++j)  // k <= 8: a fixed trip count keeps the loads independent
          if (j < d.k) {
            const float4 u = *reinterpret_cast<const float4*>(row + (size_t)j * d.D);
            v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
          }
      }
      acc[i][jv] = v.x; acc[i][jv + 1] = v.y; acc[i][jv + 2] = v.z; acc[i][jv + 3] = v.w;
    }
  }
  for (int r0 = 0; r0 < R; r0 += kBK2) {
    __syncthreads();  // the previous stage is consumed
#pragma unroll
    for (int u = 0; u < kBK2 * kBT2 / 256; ++u) {
      const int i = tid + 256 * u;
      const int row = i >> 3, kk = i & 7, m = m0 + row, r = r0 + kk;
      st.A[kk][row] = (m < d.M && r < R) ? gate_at(d, dg, du, m, r) : 0.f;
      const int kb = i >> 7, col = i & 127, n = n0 + col, rb = r0 + kb;
      float w = 0.f;
      if (rb < R && n < d.D) w = rb < d.E ? to_f32(Wr[(size_t)rb * d.D + n]) : to_f32(Wdt[(size_t)(rb - d.E) * d.D + n]);
      st.B[kb][col] = w;
    }
    __syncthreads();
    mac8x8(st, ty, tx, acc);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + ty * 8 + i;
    if (m >= d.M) continue;
#pragma unroll
    for (int jv = 0; jv < 8; jv += 4) {
      const int n = n0 + tx * 8 + jv;
      if (n < d.D)
        *reinterpret_cast<float4*>(dX + (size_t)m * d.D + n) =
            make_float4(acc[i][jv], acc[i][jv + 1], acc[i][jv + 2], acc[i][jv + 3]);
    }
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
  dw_gate_kernel<T><<<dim3(ceil_div(d.D, kGC), ceil_div(d.M, kGM), ceil_div(d.E + d.H, kGR)), 256, 0, s>>>(
      d, q.dg, q.du, (const T*)q.X, q.dW_r, q.dW_dt);
  db_kernel<<<d.H, 256, 0, s>>>(d, q.du, q.db_dt);
  dx_final_kernel<T><<<dim3(ceil_div(d.D, kBT2), ceil_div(d.M, kBT2)), 256, 0, s>>>(d, q.dxp, q.dg, q.du,
                                                                                   (const T*)q.w_r,
                                                                                   (const T*)q.w_dt, q.dX);
  count_launches(3);
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
