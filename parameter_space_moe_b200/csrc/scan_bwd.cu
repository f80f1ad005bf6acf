// Gradients of the chunked scan: reverse-mode of the single shared-transition recurrence, CUDA cores, fp32.
//
// Paper: Swimba notes, key design 1, second display equation (h_t = a_t h_{t-1} + U~_t, y_t = C~_t^T h_t);
// the notes train the model (loss function / training strategy), which needs these gradients.  For
// L = sum_t <dy_t, y_t> and 64-token sub-chunks c with cs_t the running sum of dA = dt * A from the sub-chunk
// start, H_c the state before sub-chunk c and Lam_c = dL/dH_c:
//   forward states  S_c = sum_s e^{cs_end - cs_s} sum_j Bpi_sj (x) Xs_sj,   H_{c+1} = e^{cs_end} H_c + S_c
//   adjoint states  D_c = sum_t e^{cs_t} C~_t (x) dy_t,   Lam_c = e^{cs_end} Lam_{c+1} + D_c,   Lam_nc = 0
//   per sub-chunk, with W[t][s] = e^{cs_t - cs_s} (s <= t), S1 = C~ Bpi_j^T, S2 = dy Xs_j^T:
//     dXs_sj  = sum_t W S1[t][s] dy_t + e^{cs_end - cs_s} Lam_{c+1}^T Bpi_sj
//     dBpi_sj = sum_t W S2[t][s] C~_t + e^{cs_end - cs_s} Lam_{c+1} Xs_sj
//     dC~_t   = sum_{s,j} W S2[t][s] Bpi_sj + e^{cs_t} H_c dy_t
//     q_t     = dL/dcs_t = sum_j [rowsum - colsum of W S1 S2]_t + e^{cs_t} C~_t . H_c dy_t
//               - e^{cs_end - cs_t} sum_j Bpi_tj . Lam_{c+1} Xs_tj   (+ at the last token: e^{cs_end} <Lam, H_c>
//               + sum_{s,j} e^{cs_end - cs_s} Bpi_sj . Lam_{c+1} Xs_sj)
//     dA_r    = sum_{t >= r} q_t,   d dt_r = dA_r A_h,   dA_h = sum_r dA_r dt_r,   d init = Lam_0.
// With G < H the Bpi and C~ gradients of a group's heads are summed (atomic adds into zeroed outputs).
#include "common.cuh"

namespace swimba {

namespace {
constexpr int BL = 64;     // tokens per backward sub-chunk
constexpr int kBT = 256;   // threads per CTA

struct BwdArgs {
  Dims d;
  int nc;                  // 64-token sub-chunks per sequence
  const void* bpi; const void* xs; const void* cpi;
  const float* dt; const float* A; const float* init; const float* dy;
  float* dbpi; float* dxs; float* dct; float* ddt; float* dA; float* dinit;
  float* hstart;           // [B][H][nc][N][P]  H_c
  float* work;             // [B][H][nc][N][P]  S_c, then D_c, then Lam_{c+1}
  float* cse;              // [B][H][nc]        cs at each sub-chunk's last token
};

// cs[i] = sum_{r <= i} dt_r A_h over the sub-chunk (thread 0, L <= 64)
__device__ __forceinline__ void sub_cumsum(const BwdArgs& a, int b, int h, int t0, int L, float* cs) {
  if (threadIdx.x == 0) {
    const Dims& d = a.d;
    float run = 0.f;
    for (int i = 0; i < L; ++i) {
      run += a.dt[(size_t)(b * d.T + t0 + i) * d.H + h] * a.A[h];
      cs[i] = run;
    }
  }
}

template <class S>
__device__ __forceinline__ void load_rows(const S* src, size_t m0, int k, int slot, int width, size_t stride_row,
                                          size_t col0, int L, float* dst, int ld) {
  // dst[i][c] = src[((m0 + i) * k + slot) * stride_row + col0 + c], zero past the sub-chunk
  for (int x = threadIdx.x; x < BL * width; x += blockDim.x) {
    const int i = x / width, c = x % width;
    dst[i * ld + c] = i < L ? to_f32(src[((m0 + i) * k + slot) * stride_row + col0 + c]) : 0.f;
  }
}

// 1. sub-chunk end states S_c (keys of every slot) and cs at the last token
template <class S>
__global__ void __launch_bounds__(kBT) bwd_fwd_chunk_kernel(BwdArgs a) {
  extern __shared__ float sm[];
  const Dims& d = a.d;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, g = h / d.hpg;
  const int t0 = c * BL, L = min(BL, d.T - t0);
  float* cs = sm;                    // [BL]
  float* Bs = cs + BL;               // [BL][N]
  float* Xv = Bs + BL * d.N;         // [BL][P] decay-scaled values
  sub_cumsum(a, b, h, t0, L, cs);
  __syncthreads();
  const size_t m0 = (size_t)b * d.T + t0;
  const int NP = d.N * d.P;
  constexpr int kMaxAcc = (128 * 128) / kBT;
  float acc[kMaxAcc];
  const int per = NP / kBT;  // N * P is a multiple of 256 for N, P in {16 .. 128}
#pragma unroll
  for (int r = 0; r < kMaxAcc; ++r) acc[r] = 0.f;
  for (int j = 0; j < d.k; ++j) {
    load_rows<S>((const S*)a.bpi, m0, d.k, j, d.N, d.GN, (size_t)g * d.N, L, Bs, d.N);
    load_rows<S>((const S*)a.xs, m0, d.k, j, d.P, d.HP, (size_t)h * d.P, L, Xv, d.P);
    __syncthreads();
    for (int x = threadIdx.x; x < BL * d.P; x += blockDim.x) {
      const int i = x / d.P;
      if (i < L) Xv[x] *= expf(cs[L - 1] - cs[i]);
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kMaxAcc; ++r) {
      if (r >= per) break;
      const int e = threadIdx.x + r * kBT, n = e / d.P, p = e % d.P;
      float v = acc[r];
      for (int i = 0; i < L; ++i) v = fmaf(Bs[i * d.N + n], Xv[i * d.P + p], v);
      acc[r] = v;
    }
    __syncthreads();
  }
  const size_t base = (((size_t)b * d.H + h) * a.nc + c) * NP;
#pragma unroll
  for (int r = 0; r < kMaxAcc; ++r)
    if (r < per) a.work[base + threadIdx.x + r * kBT] = acc[r];
  if (threadIdx.x == 0) a.cse[((size_t)b * d.H + h) * a.nc + c] = cs[L - 1];
}

// 2. H_c for every sub-chunk (sequential in c, parallel over (b, h, n, p))
__global__ void bwd_fwd_pass_kernel(BwdArgs a) {
  const Dims& d = a.d;
  const int NP = d.N * d.P;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  if (e >= NP) return;
  const size_t bh = (size_t)b * d.H + h;
  float v = a.init ? a.init[bh * NP + e] : 0.f;
  for (int c = 0; c < a.nc; ++c) {
    const size_t o = (bh * a.nc + c) * NP + e;
    a.hstart[o] = v;
    v = fmaf(expf(a.cse[bh * a.nc + c]), v, a.work[o]);
  }
}

// 3. D_c = sum_t e^{cs_t} C~_t (x) dy_t  (overwrites S_c)
template <class S>
__global__ void __launch_bounds__(kBT) bwd_d_kernel(BwdArgs a) {
  extern __shared__ float sm[];
  const Dims& d = a.d;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, g = h / d.hpg;
  const int t0 = c * BL, L = min(BL, d.T - t0);
  float* cs = sm;
  float* Cs = cs + BL;               // [BL][N] e^{cs_t} C~_t
  float* Dy = Cs + BL * d.N;         // [BL][P]
  sub_cumsum(a, b, h, t0, L, cs);
  const size_t m0 = (size_t)b * d.T + t0;
  for (int x = threadIdx.x; x < BL * d.N; x += blockDim.x) {
    const int i = x / d.N, n = x % d.N;
    float v = 0.f;
    if (i < L)
      for (int j = 0; j < d.k; ++j) v += to_f32(((const S*)a.cpi)[((m0 + i) * d.k + j) * d.GN + (size_t)g * d.N + n]);
    Cs[x] = v;
  }
  for (int x = threadIdx.x; x < BL * d.P; x += blockDim.x) {
    const int i = x / d.P, p = x % d.P;
    Dy[x] = i < L ? a.dy[(m0 + i) * d.HP + (size_t)h * d.P + p] : 0.f;
  }
  __syncthreads();
  for (int x = threadIdx.x; x < BL * d.N; x += blockDim.x) {
    const int i = x / d.N;
    if (i < L) Cs[x] *= expf(cs[i]);
  }
  __syncthreads();
  const int NP = d.N * d.P;
  const size_t base = (((size_t)b * d.H + h) * a.nc + c) * NP;
  for (int e = threadIdx.x; e < NP; e += blockDim.x) {
    const int n = e / d.P, p = e % d.P;
    float v = 0.f;
    for (int i = 0; i < L; ++i) v = fmaf(Cs[i * d.N + n], Dy[i * d.P + p], v);
    a.work[base + e] = v;
  }
}

// 4. Lam_{c+1} for every sub-chunk (into work, replacing D_c), and d init = Lam_0
__global__ void bwd_adj_pass_kernel(BwdArgs a) {
  const Dims& d = a.d;
  const int NP = d.N * d.P;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  if (e >= NP) return;
  const size_t bh = (size_t)b * d.H + h;
  float lam = 0.f;
  for (int c = a.nc - 1; c >= 0; --c) {
    const size_t o = (bh * a.nc + c) * NP + e;
    const float Dc = a.work[o];
    a.work[o] = lam;
    lam = fmaf(expf(a.cse[bh * a.nc + c]), lam, Dc);
  }
  if (a.dinit) a.dinit[bh * NP + e] = lam;
}

// Shared-memory plan of the gradient kernel (floats): per sub-chunk C~, dy, then per slot keys, values,
// the two score tiles, and the end adjoint Lam_{c+1} (with H_c first, for the carried-state terms).
struct GradSmem {
  int N, P, ldS;
  size_t cs, eend, q, bv, red, C, Dy, B, X, S1, S2, Lam, total;
  __host__ __device__ GradSmem(int n, int p) : N(n), P(p), ldS(BL + 1) {
    size_t o = 0;
    cs = o; o += BL;
    eend = o; o += BL;
    q = o; o += BL;
    bv = o; o += BL;
    red = o; o += 4;
    C = o; o += (size_t)BL * N;
    Dy = o; o += (size_t)BL * P;
    B = o; o += (size_t)BL * N;
    X = o; o += (size_t)BL * P;
    S1 = o; o += (size_t)BL * ldS;
    S2 = o; o += (size_t)BL * ldS;
    Lam = o; o += (size_t)N * P;
    total = o;
  }
};

// 5. the per-sub-chunk gradients
template <class S>
__global__ void __launch_bounds__(kBT) bwd_grad_kernel(BwdArgs a) {
  extern __shared__ float sm[];
  const Dims& d = a.d;
  const GradSmem Ls(d.N, d.P);
  const int N = d.N, P = d.P, ldS = Ls.ldS;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, g = h / d.hpg;
  const int t0 = c * BL, L = min(BL, d.T - t0);
  float* cs = sm + Ls.cs;
  float* eend = sm + Ls.eend;
  float* q = sm + Ls.q;
  float* bv = sm + Ls.bv;
  float* red = sm + Ls.red;
  float* C = sm + Ls.C;
  float* Dy = sm + Ls.Dy;
  float* Bs = sm + Ls.B;
  float* Xs = sm + Ls.X;
  float* S1 = sm + Ls.S1;
  float* S2 = sm + Ls.S2;
  float* Lam = sm + Ls.Lam;
  const int tid = threadIdx.x;
  const size_t m0 = (size_t)b * d.T + t0;
  const size_t bh = (size_t)b * d.H + h;
  const int NP = N * P;
  const size_t sbase = (bh * a.nc + c) * NP;

  sub_cumsum(a, b, h, t0, L, cs);
  for (int i = tid; i < BL; i += blockDim.x) { q[i] = 0.f; bv[i] = 0.f; }
  if (tid < 4) red[tid] = 0.f;
  for (int x = tid; x < BL * N; x += blockDim.x) {
    const int i = x / N, n = x % N;
    float v = 0.f;
    if (i < L)
      for (int j = 0; j < d.k; ++j) v += to_f32(((const S*)a.cpi)[((m0 + i) * d.k + j) * d.GN + (size_t)g * N + n]);
    C[x] = v;
  }
  for (int x = tid; x < BL * P; x += blockDim.x) {
    const int i = x / P, p = x % P;
    Dy[x] = i < L ? a.dy[(m0 + i) * d.HP + (size_t)h * P + p] : 0.f;
  }
  // H_c into the Lam buffer first; e^{cs_end} <Lam_{c+1}, H_c> on the way
  float part = 0.f;
  for (int e = tid; e < NP; e += blockDim.x) {
    const float hv = a.hstart[sbase + e];
    Lam[e] = hv;
    part = fmaf(a.work[sbase + e], hv, part);
  }
  atomicAdd(&red[0], part);
  __syncthreads();
  const float cs_end = cs[L - 1];
  for (int i = tid; i < BL; i += blockDim.x) eend[i] = i < L ? expf(cs_end - cs[i]) : 0.f;
  // carried-state terms: dC~_t = e^{cs_t} H_c dy_t (kept per thread over the slots), q_t = C~_t . that
  constexpr int kMaxPer = (BL * 128) / kBT;
  float dC[kMaxPer];
  const int perC = (BL * N) / kBT;
#pragma unroll
  for (int r = 0; r < kMaxPer; ++r) {
    if (r >= perC) break;
    const int x = tid + r * kBT, i = x / N, n = x % N;
    float v = 0.f;
    if (i < L) {
      for (int p = 0; p < P; ++p) v = fmaf(Lam[n * P + p], Dy[i * P + p], v);
      v *= expf(cs[i]);
    }
    dC[r] = v;
    if (i < L) atomicAdd(&q[i], C[i * N + n] * v);
  }
  __syncthreads();
  // the end adjoint Lam_{c+1}
  for (int e = tid; e < NP; e += blockDim.x) Lam[e] = a.work[sbase + e];
  __syncthreads();

  for (int j = 0; j < d.k; ++j) {
    load_rows<S>((const S*)a.bpi, m0, d.k, j, N, d.GN, (size_t)g * N, L, Bs, N);
    load_rows<S>((const S*)a.xs, m0, d.k, j, P, d.HP, (size_t)h * P, L, Xs, P);
    __syncthreads();
    // score tiles with the causal decay: K1 = W S1 (into S1), K2 = W S2 (into S2); M = W S1 S2 into q
    for (int x = tid; x < BL * BL; x += blockDim.x) {
      const int t = x / BL, s = x % BL;
      float k1 = 0.f, k2 = 0.f;
      if (s <= t && t < L) {
        float s1 = 0.f, s2 = 0.f;
        for (int n = 0; n < N; ++n) s1 = fmaf(C[t * N + n], Bs[s * N + n], s1);
        for (int p = 0; p < P; ++p) s2 = fmaf(Dy[t * P + p], Xs[s * P + p], s2);
        const float w = expf(cs[t] - cs[s]);
        k1 = w * s1;
        k2 = w * s2;
        const float m = k1 * s2;
        atomicAdd(&q[t], m);
        atomicAdd(&q[s], -m);
      }
      S1[t * ldS + s] = k1;
      S2[t * ldS + s] = k2;
    }
    __syncthreads();
    // dXs_s = sum_t K1[t][s] dy_t + e^{cs_end - cs_s} Lam^T B_s
    for (int x = tid; x < BL * P; x += blockDim.x) {
      const int s = x / P, p = x % P;
      if (s >= L) continue;
      float v = 0.f, u = 0.f;
      for (int t = s; t < L; ++t) v = fmaf(S1[t * ldS + s], Dy[t * P + p], v);
      for (int n = 0; n < N; ++n) u = fmaf(Lam[n * P + p], Bs[s * N + n], u);
      a.dxs[((m0 + s) * d.k + j) * d.HP + (size_t)h * P + p] = fmaf(eend[s], u, v);
    }
    // dBpi_s = sum_t K2[t][s] C~_t + e^{cs_end - cs_s} Lam x_s;  bv_s += B_s . Lam x_s
    for (int x = tid; x < BL * N; x += blockDim.x) {
      const int s = x / N, n = x % N;
      if (s >= L) continue;
      float v = 0.f, u = 0.f;
      for (int t = s; t < L; ++t) v = fmaf(S2[t * ldS + s], C[t * N + n], v);
      for (int p = 0; p < P; ++p) u = fmaf(Lam[n * P + p], Xs[s * P + p], u);
      atomicAdd(&a.dbpi[((m0 + s) * d.k + j) * d.GN + (size_t)g * N + n], fmaf(eend[s], u, v));
      atomicAdd(&bv[s], Bs[s * N + n] * u);
    }
    // dC~_t += sum_{s <= t} K2[t][s] B_s
#pragma unroll
    for (int r = 0; r < kMaxPer; ++r) {
      if (r >= perC) break;
      const int x = tid + r * kBT, t = x / N, n = x % N;
      if (t >= L) continue;
      float v = dC[r];
      for (int s = 0; s <= t; ++s) v = fmaf(S2[t * ldS + s], Bs[s * N + n], v);
      dC[r] = v;
    }
    __syncthreads();
    // q_t -= e^{cs_end - cs_t} bv_t, and the last token takes sum_s e^{cs_end - cs_s} bv_s
    if (tid < L) {
      const float e = eend[tid] * bv[tid];
      atomicAdd(&q[tid], -e);
      atomicAdd(&red[1], e);
      bv[tid] = 0.f;
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < kMaxPer; ++r) {
    if (r >= perC) break;
    const int x = tid + r * kBT, t = x / N, n = x % N;
    if (t < L) atomicAdd(&a.dct[(m0 + t) * d.GN + (size_t)g * N + n], dC[r]);
  }
  if (tid == 0) {
    q[L - 1] += expf(cs_end) * red[0] + red[1];
    // dA_r = sum_{t >= r} q_t;  d dt_r = dA_r A_h;  dA_h += sum_r dA_r dt_r
    float run = 0.f, dAh = 0.f;
    const float Ah = a.A[h];
    for (int r = L - 1; r >= 0; --r) {
      run += q[r];
      const size_t o = (m0 + r) * d.H + h;
      a.ddt[o] = run * Ah;
      dAh = fmaf(run, a.dt[o], dAh);
    }
    atomicAdd(&a.dA[h], dAh);
  }
}

template <class S>
cudaError_t launch_bwd_typed(const BwdArgs& a, cudaStream_t s) {
  const Dims& d = a.d;
  const dim3 grid(a.nc, d.H, d.Bsz);
  const size_t sm1 = (BL + (size_t)BL * d.N + (size_t)BL * d.P) * 4;
  cudaError_t e = set_max_dynamic_smem((const void*)bwd_fwd_chunk_kernel<S>, sm1);
  if (e != cudaSuccess) return e;
  bwd_fwd_chunk_kernel<S><<<grid, kBT, sm1, s>>>(a);
  const dim3 pgrid(ceil_div(d.N * d.P, kBT), d.H, d.Bsz);
  bwd_fwd_pass_kernel<<<pgrid, kBT, 0, s>>>(a);
  e = set_max_dynamic_smem((const void*)bwd_d_kernel<S>, sm1);
  if (e != cudaSuccess) return e;
  bwd_d_kernel<S><<<grid, kBT, sm1, s>>>(a);
  bwd_adj_pass_kernel<<<pgrid, kBT, 0, s>>>(a);
  const size_t sm5 = GradSmem(d.N, d.P).total * 4;
  e = set_max_dynamic_smem((const void*)bwd_grad_kernel<S>, sm5);
  if (e != cudaSuccess) return e;
  bwd_grad_kernel<S><<<grid, kBT, sm5, s>>>(a);
  count_launches(5);
  return cudaGetLastError();
}
}  // namespace

int scan_bwd_subchunks(const Dims& d) { return ceil_div(d.T, BL); }

// Shared memory of the gradient kernel for these dims (bytes); the entry point refuses shapes above the
// per-CTA limit.
size_t scan_bwd_smem(const Dims& d) { return GradSmem(d.N, d.P).total * 4; }

cudaError_t launch_scan_bwd(const Dims& d, const void* bpi, const void* xs, const void* cpi, const float* dt,
                            const float* A, const float* init, const float* dy, float* dbpi, float* dxs, float* dct,
                            float* ddt, float* dA, float* dinit, float* hstart, float* work, float* cse,
                            cudaStream_t s) {
  BwdArgs a{d, scan_bwd_subchunks(d), bpi, xs, cpi, dt, A, init, dy, dbpi, dxs, dct, ddt, dA, dinit,
            hstart, work, cse};
  // the Bpi, C~ and A gradients are accumulated
  cudaError_t e = cudaMemsetAsync(dbpi, 0, (size_t)d.M * d.k * d.GN * 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(dct, 0, (size_t)d.M * d.GN * 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(dA, 0, (size_t)d.H * 4, s);
  if (e != cudaSuccess) return e;
  return d.dtype == SWIMBA_BF16 ? launch_bwd_typed<__half>(a, s) : launch_bwd_typed<float>(a, s);
}

}  // namespace swimba
