// Gradients of the chunked scan: reverse-mode of the single shared-transition recurrence, fp32 values and
// accumulation (the sub-chunk end states and adjoint sources on the tensor cores for fp16 streams with
// N = 128, everything else on CUDA cores).
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
// With G < H the Bpi and C~ gradients of a group's heads are summed (atomic adds into zeroed outputs); with
// G = H every output element is written by exactly one CTA.
#include "tc_common.cuh"

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
  unsigned* st;            // device status word (bounded waits of the tensor-core state kernels)
};

// cs[i] = sum_{r <= i} dt_r A_h over the sub-chunk (warp 0: two tokens per lane, shuffle scans; L <= 64)
__device__ __forceinline__ void sub_cumsum(const BwdArgs& a, int b, int h, int t0, int L, float* cs) {
  if (threadIdx.x < 32) {
    const Dims& d = a.d;
    const int lane = threadIdx.x;
    const float Ah = a.A[h];
    float v0 = lane < L ? a.dt[(size_t)(b * d.T + t0 + lane) * d.H + h] * Ah : 0.f;
    float v1 = lane + 32 < L ? a.dt[(size_t)(b * d.T + t0 + lane + 32) * d.H + h] * Ah : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u0 = __shfl_up_sync(0xffffffffu, v0, o), u1 = __shfl_up_sync(0xffffffffu, v1, o);
      if (lane >= o) { v0 += u0; v1 += u1; }
    }
    const float first = __shfl_sync(0xffffffffu, v0, 31);
    cs[lane] = v0;
    cs[lane + 32] = v1 + first;
  }
}

// acc[i][jj] += sum_{k < K} X(k, r_i) Y(k, c_jj) for rows r_i = ty + 16 i (i < 4) and columns c_jj = tx + 16 jj
// (jj < nj); X(k, r) = X[k * xk + r * xr], Y(k, c) = Y[k * yk + c * yc].  A 16 x 16 thread grid over a 64-row
// output, every thread with 4 x nj independent accumulators.
template <int MJ, int MI = 4>
__device__ __forceinline__ void tile_mac(float (&acc)[MI][MJ], int nj, int K, const float* X, int xk, int xr,
                                         const float* Y, int yk, int yc, int ty, int tx, int ni = MI) {
#pragma unroll 8
  for (int k = 0; k < K; ++k) {
    float xv[MI], yv[MJ];
#pragma unroll
    for (int i = 0; i < MI; ++i) xv[i] = i < ni ? X[k * xk + (ty + 16 * i) * xr] : 0.f;
#pragma unroll
    for (int jj = 0; jj < MJ; ++jj) yv[jj] = jj < nj ? Y[k * yk + (tx + 16 * jj) * yc] : 0.f;
#pragma unroll
    for (int i = 0; i < MI; ++i)
#pragma unroll
      for (int jj = 0; jj < MJ; ++jj) acc[i][jj] = fmaf(xv[i], yv[jj], acc[i][jj]);
  }
}

__device__ __forceinline__ void widen(const uint4& q, float (&f)[8]) {
  const __half2* h = reinterpret_cast<const __half2*>(&q);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 v = __half22float2(h[e]);
    f[2 * e] = v.x;
    f[2 * e + 1] = v.y;
  }
}
__device__ __forceinline__ void widen(const uint4& q, float (&f)[4]) {
  const float* v = reinterpret_cast<const float*>(&q);
#pragma unroll
  for (int e = 0; e < 4; ++e) f[e] = v[e];
}

// dst[i][c] = src[((m0 + i) * k + slot) * stride_row + col0 + c] for i < BL, c < width, zero past the
// sub-chunk; 16-byte loads (width, stride_row and col0 are multiples of 8 elements, the rows 16-byte aligned)
template <class S>
__device__ __forceinline__ void load_rows(const S* src, size_t m0, int k, int slot, int width, size_t stride_row,
                                          size_t col0, int L, float* dst, int ld) {
  constexpr int V = 16 / sizeof(S);
  const int per_row = width / V;
  for (int x = threadIdx.x; x < BL * per_row; x += blockDim.x) {
    const int i = x / per_row, c = (x - i * per_row) * V;
    float f[V];
    if (i < L) {
      widen(*reinterpret_cast<const uint4*>(src + ((m0 + i) * k + slot) * stride_row + col0 + c), f);
    } else {
#pragma unroll
      for (int e = 0; e < V; ++e) f[e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < V; ++e) dst[i * ld + c + e] = f[e];
  }
}

// dst[i][c] = sum_{j < k} src[((m0 + i) * k + j) * stride_row + col0 + c] (C~ from the per-slot readouts)
template <class S>
__device__ __forceinline__ void load_rows_sum(const S* src, size_t m0, int k, int width, size_t stride_row,
                                              size_t col0, int L, float* dst, int ld) {
  constexpr int V = 16 / sizeof(S);
  const int per_row = width / V;
  for (int x = threadIdx.x; x < BL * per_row; x += blockDim.x) {
    const int i = x / per_row, c = (x - i * per_row) * V;
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    if (i < L) {
      for (int j = 0; j < k; ++j) {
        float f[V];
        widen(*reinterpret_cast<const uint4*>(src + ((m0 + i) * k + j) * stride_row + col0 + c), f);
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] += f[e];
      }
    }
#pragma unroll
    for (int e = 0; e < V; ++e) dst[i * ld + c + e] = acc[e];
  }
}

// 1. sub-chunk end states S_c (keys of every slot) and cs at the last token.  PJ = P / 16 column groups per
// thread (a compile-time count, so no FMA runs on a padding column).
template <class S, int PJ>
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
  // thread (ty, tx) of a 16 x 16 grid holds S_c[n][p] for n = ty + 16 i, p = tx + 16 jj
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4, ni = d.N / 16;
  float acc[8][PJ];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int jj = 0; jj < PJ; ++jj) acc[i][jj] = 0.f;
  for (int j = 0; j < d.k; ++j) {
    load_rows<S>((const S*)a.bpi, m0, d.k, j, d.N, d.GN, (size_t)g * d.N, L, Bs, d.N);
    load_rows<S>((const S*)a.xs, m0, d.k, j, d.P, d.HP, (size_t)h * d.P, L, Xv, d.P);
    __syncthreads();
    for (int x = threadIdx.x; x < BL * d.P; x += blockDim.x) {
      const int i = x / d.P;
      if (i < L) Xv[x] *= expf(cs[L - 1] - cs[i]);
    }
    __syncthreads();
    tile_mac<PJ, 8>(acc, PJ, L, Bs, d.N, 1, Xv, d.P, 1, ty, tx, ni);
    __syncthreads();
  }
  const size_t base = (((size_t)b * d.H + h) * a.nc + c) * NP;
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int jj = 0; jj < PJ; ++jj)
      if (i < ni) a.work[base + (size_t)(ty + 16 * i) * d.P + tx + 16 * jj] = acc[i][jj];
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
template <class S, int PJ>
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
  load_rows_sum<S>((const S*)a.cpi, m0, d.k, d.N, d.GN, (size_t)g * d.N, L, Cs, d.N);
  load_rows<float>(a.dy, m0, 1, 0, d.P, d.HP, (size_t)h * d.P, L, Dy, d.P);
  __syncthreads();
  for (int x = threadIdx.x; x < BL * d.N; x += blockDim.x) {
    const int i = x / d.N;
    if (i < L) Cs[x] *= expf(cs[i]);
  }
  __syncthreads();
  const int NP = d.N * d.P;
  const size_t base = (((size_t)b * d.H + h) * a.nc + c) * NP;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4, ni = d.N / 16;
  float acc[8][PJ];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int jj = 0; jj < PJ; ++jj) acc[i][jj] = 0.f;
  tile_mac<PJ, 8>(acc, PJ, L, Cs, d.N, 1, Dy, d.P, 1, ty, tx, ni);
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int jj = 0; jj < PJ; ++jj)
      if (i < ni) a.work[base + (size_t)(ty + 16 * i) * d.P + tx + 16 * jj] = acc[i][jj];
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
  float Dnext = a.work[(bh * a.nc + a.nc - 1) * NP + e];
  for (int c = a.nc - 1; c >= 0; --c) {
    const size_t o = (bh * a.nc + c) * NP + e;
    const float Dc = Dnext;
    if (c > 0) Dnext = a.work[o - NP];
    a.work[o] = lam;
    lam = fmaf(expf(a.cse[bh * a.nc + c]), lam, Dc);
  }
  if (a.dinit) a.dinit[bh * NP + e] = lam;
}

// 1'/3'. The end states S_c and the adjoint sources D_c on the tensor cores (fp16 streams, N = 128,
// P in {64, 128}).  Both are [N x P] = A^T B over the sub-chunk's tokens:
//   S_c = sum_j Bpi_j^T (e^{cs_end - cs} * Xs_j),   D_c = sum_j Cpi_j^T (e^{cs} * dy)
// A (the fp16 stream rows, exact) is M = n by K = token, read MN-major; B is formed in fp32 and split into two
// fp16 halves hi + lo (two MMAs into one fp32 accumulator: about 2^-22 relative); dy first takes a
// power-of-two scale that puts the tile's largest value near 2^15 (exact, undone on the result), so the
// split stays inside fp16's range.  One CTA of 4 warps per (sequence, head, 64-token sub-chunk); operands
// are staged slot by slot in 128-byte-swizzled shared memory by plain 16-byte loads; the accumulator sits in
// P TMEM columns.
constexpr uint32_t kTcBlk = BL * 128;  // one 64-wide MN block of 64 K rows of 128 bytes
// dynamic shared memory of the tensor-core state kernels: alignment slack, A, B hi and lo, cs, scale
// partials, mbarrier, TMEM slot and abort flag
inline size_t states_tc_smem(int P) { return 1024 + 2 * kTcBlk + 2 * (size_t)(P / 64) * kTcBlk + (BL + 4) * 4 + 24; }
template <bool kD, int kP>
__global__ void __launch_bounds__(128) bwd_states_tc_kernel(BwdArgs a) {
  extern __shared__ uint8_t smraw[];
  const uint32_t raw = tc::smem_u32(smraw);
  uint8_t* sm = smraw + (((raw + 1023u) & ~1023u) - raw);
  const Dims& d = a.d;
  constexpr int N = 128, PB = kP / 64;
  constexpr int kAU = BL * 16 / 128;        // 16-byte A chunks per thread (8)
  constexpr int kBU = BL * (kP / 8) / 128;  // 8-column B groups per thread (4 or 8)
  uint8_t* As = sm;                          // 2 MN blocks (n 0..63, 64..127)
  uint8_t* Bhi = As + 2 * kTcBlk;            // PB MN blocks
  uint8_t* Blo = Bhi + PB * kTcBlk;
  float* cs = reinterpret_cast<float*>(Blo + PB * kTcBlk);  // [BL]
  float* red = cs + BL;                                     // [4]
  uint64_t* bar = reinterpret_cast<uint64_t*>(red + 4);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, g = h / d.hpg;
  const int t0 = c * BL, L = min(BL, d.T - t0);
  const size_t m0 = (size_t)b * d.T + t0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  sub_cumsum(a, b, h, t0, L, cs);
  if (tid == 0) {
    tc::mbar_init(bar, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) { tc::tmem_alloc(tslot, (uint32_t)kP); tc::tmem_relinquish(); }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;
  const float cs_end = cs[L - 1];
  // B: row s (token), columns p0 .. p0+7 as one 16-byte fp16 chunk of each half
  auto put_b = [&](int s, int p0, const float (&v)[8]) {
    uint4 uh, ul;
    __half2* hh = reinterpret_cast<__half2*>(&uh);
    __half2* hl = reinterpret_cast<__half2*>(&ul);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      hh[e] = __floats2half2_rn(v[2 * e], v[2 * e + 1]);
      const float2 f = __half22float2(hh[e]);
      hl[e] = __floats2half2_rn(v[2 * e] - f.x, v[2 * e + 1] - f.y);
    }
    const uint32_t off = (p0 >> 6) * kTcBlk + tc::sw128_chunk(s, (p0 & 63) >> 3);
    *reinterpret_cast<uint4*>(Bhi + off) = uh;
    *reinterpret_cast<uint4*>(Blo + off) = ul;
  };
  int sc = 0;  // D_c: power-of-two scale of e^{cs} dy
  if constexpr (kD) {
    // e^{cs_t} dy_t for this thread's groups, all loads issued before any use
    float v[kBU][8];
#pragma unroll
    for (int u = 0; u < kBU; ++u) {
      const int x = tid + 128 * u, s = x / (kP / 8), p0 = (x % (kP / 8)) * 8;
      if (s < L) {
        const float* src = a.dy + (m0 + s) * d.HP + (size_t)h * kP + p0;
        const float4 u0 = *reinterpret_cast<const float4*>(src), u1 = *reinterpret_cast<const float4*>(src + 4);
        v[u][0] = u0.x; v[u][1] = u0.y; v[u][2] = u0.z; v[u][3] = u0.w;
        v[u][4] = u1.x; v[u][5] = u1.y; v[u][6] = u1.z; v[u][7] = u1.w;
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) v[u][q] = 0.f;
      }
    }
    float mx = 0.f;
#pragma unroll
    for (int u = 0; u < kBU; ++u) {
      const int s = (tid + 128 * u) / (kP / 8);
      const float e = s < L ? expf(cs[s]) : 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        v[u][q] *= e;
        mx = fmaxf(mx, fabsf(v[u][q]));
      }
    }
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    if (mx > 0.f && mx < 3.0e38f) {
      int ex;
      frexpf(mx, &ex);
      sc = 15 - ex;
    }
    // B = e^{cs_t} dy_t 2^sc (the scale applies to the product, bounded by the tile's maximum), every slot
#pragma unroll
    for (int u = 0; u < kBU; ++u) {
      const int x = tid + 128 * u, s = x / (kP / 8), p0 = (x % (kP / 8)) * 8;
#pragma unroll
      for (int q = 0; q < 8; ++q) v[u][q] = ldexpf(v[u][q], sc);
      put_b(s, p0, v[u]);
    }
  }
  constexpr uint32_t idesc = tc::idesc_f16(128, kP, /*bf16=*/false, /*a_mn=*/true, /*b_mn=*/true);
  const __half* Asrc = reinterpret_cast<const __half*>(kD ? a.cpi : a.bpi);
  uint32_t phase = 0;
  bool ok = true;
  for (int j = 0; j < d.k && ok; ++j) {
    // A_j: the slot's N-wide stream rows (16 chunks of 8 per row); B_j (end states): e^{cs_end - cs_s} Xs_j.
    // All of this thread's loads are issued before the first store.
    uint4 av[kAU];
#pragma unroll
    for (int u = 0; u < kAU; ++u) {
      const int x = tid + 128 * u, s = x >> 4, ch = x & 15;
      av[u] = s < L ? *reinterpret_cast<const uint4*>(Asrc + ((m0 + s) * d.k + j) * d.GN + (size_t)g * N + ch * 8)
                    : make_uint4(0u, 0u, 0u, 0u);
    }
    uint4 xv[kD ? 1 : kBU];
    if constexpr (!kD) {
#pragma unroll
      for (int u = 0; u < kBU; ++u) {
        const int x = tid + 128 * u, s = x / (kP / 8), p0 = (x % (kP / 8)) * 8;
        xv[u] = s < L ? *reinterpret_cast<const uint4*>(reinterpret_cast<const __half*>(a.xs) +
                                                        ((m0 + s) * d.k + j) * d.HP + (size_t)h * kP + p0)
                      : make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < kAU; ++u) {
      const int x = tid + 128 * u, s = x >> 4, ch = x & 15;
      *reinterpret_cast<uint4*>(As + (ch >> 3) * kTcBlk + tc::sw128_chunk(s, ch & 7)) = av[u];
    }
    if constexpr (!kD) {
#pragma unroll
      for (int u = 0; u < kBU; ++u) {
        const int x = tid + 128 * u, s = x / (kP / 8), p0 = (x % (kP / 8)) * 8;
        const float e = s < L ? expf(cs_end - cs[s]) : 0.f;
        const __half2* hq = reinterpret_cast<const __half2*>(&xv[u]);
        float v[8];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const float2 f = __half22float2(hq[e2]);
          v[2 * e2] = e * f.x;
          v[2 * e2 + 1] = e * f.y;
        }
        put_b(s, p0, v);
      }
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0) {
      const uint32_t sa = tc::smem_u32(As), sh = tc::smem_u32(Bhi), sl = tc::smem_u32(Blo);
#pragma unroll
      for (int part = 0; part < 2; ++part)
#pragma unroll
        for (int kk = 0; kk < BL / 16; ++kk)
          tc::mma_f16(tmem, tc::sdesc_mnmajor_sw128(sa + kk * 2048, kTcBlk),
                      tc::sdesc_mnmajor_sw128((part ? sl : sh) + kk * 2048, kTcBlk), idesc,
                      (j | part | kk) != 0);
      tc::mma_commit(bar);
    }
    // the slot's MMAs read the staged operands: wait before the next slot overwrites them
    ok = tc::mbar_wait(bar, phase, abort_flag);
    phase ^= 1u;
    tc::fence_after_sync();
  }
  if (!ok && lane == 0) atomicOr(a.st, ST_TIMEOUT);
  // TMEM lane n (warp w: lanes 32w ..) holds row n of the [N x P] result
  const size_t base = (((size_t)b * d.H + h) * a.nc + c) * (size_t)N * kP;
  const int n = 32 * warp + lane;
#pragma unroll
  for (int c0 = 0; c0 < kP; c0 += 32) {
    if (!ok) break;
    uint32_t r[32];
    tc::tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0, r);
    tc::tmem_ld_wait(r);
    float* dst = a.work + base + (size_t)n * kP + c0;
#pragma unroll
    for (int i = 0; i < 32; i += 4)
      *reinterpret_cast<float4*>(dst + i) =
          make_float4(ldexpf(__uint_as_float(r[i]), -sc), ldexpf(__uint_as_float(r[i + 1]), -sc),
                      ldexpf(__uint_as_float(r[i + 2]), -sc), ldexpf(__uint_as_float(r[i + 3]), -sc));
  }
  if (!kD && tid == 0) a.cse[((size_t)b * d.H + h) * a.nc + c] = cs_end;
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, (uint32_t)kP);
  }
}

// Shared-memory plan of the gradient kernel (floats): per sub-chunk C~, dy, then per slot keys, values,
// the two score tiles, and the end adjoint Lam_{c+1} (with H_c first, for the carried-state terms).  Rows of
// N or P floats are padded by one so that column walks across rows hit distinct banks.
struct GradSmem {
  int N, P, ldN, ldP;
  size_t cs, eend, q, bv, red, C, Dy, B, X, S1, S2, Lam, total;
  __host__ __device__ GradSmem(int n, int p) : N(n), P(p), ldN(n + 1), ldP(p + 1) {
    size_t o = 0;
    cs = o; o += BL;
    eend = o; o += BL;
    q = o; o += BL;
    bv = o; o += BL;
    red = o; o += 4;
    C = o; o += (size_t)BL * ldN;
    Dy = o; o += (size_t)BL * ldP;
    B = o; o += (size_t)BL * ldN;
    X = o; o += (size_t)BL * ldP;
    S1 = o; o += (size_t)BL * BL;
    S2 = o; o += (size_t)BL * BL;
    Lam = o; o += (size_t)N * ldP;
    total = o;
  }
};

// 5. the per-sub-chunk gradients (PJ = P / 16 column groups of the dXs tile, compile-time)
template <class S, int PJ>
__global__ void __launch_bounds__(kBT) bwd_grad_kernel(BwdArgs a) {
  extern __shared__ float sm[];
  const Dims& d = a.d;
  const GradSmem Ls(d.N, d.P);
  const int N = d.N, P = d.P, ldN = Ls.ldN, ldP = Ls.ldP;
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
  load_rows_sum<S>((const S*)a.cpi, m0, d.k, N, d.GN, (size_t)g * N, L, C, ldN);
  load_rows<float>(a.dy, m0, 1, 0, P, d.HP, (size_t)h * P, L, Dy, ldP);
  // H_c into the Lam buffer first; e^{cs_end} <Lam_{c+1}, H_c> on the way (16-byte loads of both)
  float part = 0.f;
  for (int e = 4 * tid; e < NP; e += 4 * blockDim.x) {
    const float4 hv = *reinterpret_cast<const float4*>(a.hstart + sbase + e);
    const float4 lv = *reinterpret_cast<const float4*>(a.work + sbase + e);
    float* dst = Lam + (e / P) * ldP + e % P;
    dst[0] = hv.x; dst[1] = hv.y; dst[2] = hv.z; dst[3] = hv.w;
    part = fmaf(lv.x, hv.x, fmaf(lv.y, hv.y, fmaf(lv.z, hv.z, fmaf(lv.w, hv.w, part))));
  }
  atomicAdd(&red[0], part);
  __syncthreads();
  const float cs_end = cs[L - 1];
  for (int i = tid; i < BL; i += blockDim.x) eend[i] = i < L ? expf(cs_end - cs[i]) : 0.f;
  // carried-state terms: dC~_t = e^{cs_t} H_c dy_t, kept per thread over the slots as a 4 x N/16 tile of
  // (t = ty + 16 i, n = tx + 16 jj); q_t = C~_t . that (the 16 lanes of a half-warp share t)
  const int tx = tid & 15, ty = tid >> 4;
  const int nN = N / 16;
  float dC[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) dC[i][jj] = 0.f;
  tile_mac<8>(dC, nN, P, Dy, 1, ldP, Lam, 1, ldP, ty, tx);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = ty + 16 * i;
    const float e = t < L ? expf(cs[t]) : 0.f;
    float qp = 0.f;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      if (jj >= nN) break;
      dC[i][jj] *= e;
      qp = fmaf(C[t * ldN + tx + 16 * jj], dC[i][jj], qp);
    }
    for (int o = 8; o > 0; o >>= 1) qp += __shfl_xor_sync(0xffffffffu, qp, o);
    if (tx == 0 && t < L) atomicAdd(&q[t], qp);
  }
  __syncthreads();
  // the end adjoint Lam_{c+1}
  for (int e = 4 * tid; e < NP; e += 4 * blockDim.x) {
    const float4 lv = *reinterpret_cast<const float4*>(a.work + sbase + e);
    float* dst = Lam + (e / P) * ldP + e % P;
    dst[0] = lv.x; dst[1] = lv.y; dst[2] = lv.z; dst[3] = lv.w;
  }
  __syncthreads();

  for (int j = 0; j < d.k; ++j) {
    load_rows<S>((const S*)a.bpi, m0, d.k, j, N, d.GN, (size_t)g * N, L, Bs, ldN);
    load_rows<S>((const S*)a.xs, m0, d.k, j, P, d.HP, (size_t)h * P, L, Xs, ldP);
    __syncthreads();
    // score tiles with the causal decay, 4 x 4 (t, s) pairs per thread: K1 = W S1 (into S1), K2 = W S2 (into S2);
    // M = W S1 S2 adds its row sums to q and takes its column sums from it
    {
      const int tx = tid & 15, ty = tid >> 4;
      float s1[4][4], s2[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) { s1[i][jj] = 0.f; s2[i][jj] = 0.f; }
#pragma unroll 8
      for (int n = 0; n < N; ++n) {
        float cv[4], bw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) { cv[i] = C[(ty + 16 * i) * ldN + n]; bw[i] = Bs[(tx + 16 * i) * ldN + n]; }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) s1[i][jj] = fmaf(cv[i], bw[jj], s1[i][jj]);
      }
#pragma unroll 8
      for (int p = 0; p < P; ++p) {
        float dv[4], xv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) { dv[i] = Dy[(ty + 16 * i) * ldP + p]; xv[i] = Xs[(tx + 16 * i) * ldP + p]; }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) s2[i][jj] = fmaf(dv[i], xv[jj], s2[i][jj]);
      }
      float rowp[4] = {0.f, 0.f, 0.f, 0.f}, colp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int t = ty + 16 * i, s = tx + 16 * jj;
          float k1 = 0.f, k2 = 0.f;
          if (s <= t && t < L) {
            const float w = expf(cs[t] - cs[s]);
            k1 = w * s1[i][jj];
            k2 = w * s2[i][jj];
            const float m = k1 * s2[i][jj];
            rowp[i] += m;
            colp[jj] += m;
          }
          S1[t * BL + s] = k1;
          S2[t * BL + s] = k2;
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        atomicAdd(&q[ty + 16 * i], rowp[i]);
        atomicAdd(&q[tx + 16 * i], -colp[i]);
      }
    }
    __syncthreads();
    // dXs_s = e^{cs_end - cs_s} Lam^T B_s + sum_t K1[t][s] dy_t   (tile of s = ty + 16 i, p = tx + 16 jj)
    {
      float ax[4][PJ];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < PJ; ++jj) ax[i][jj] = 0.f;
      tile_mac<PJ>(ax, PJ, N, Bs, 1, ldN, Lam, ldP, 1, ty, tx);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < PJ; ++jj) ax[i][jj] *= eend[ty + 16 * i];
      tile_mac<PJ>(ax, PJ, L, S1, BL, 1, Dy, ldP, 1, ty, tx);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int s = ty + 16 * i;
        if (s >= L) continue;
#pragma unroll
        for (int jj = 0; jj < PJ; ++jj) a.dxs[((m0 + s) * d.k + j) * d.HP + (size_t)h * P + tx + 16 * jj] = ax[i][jj];
      }
    }
    float acc[4][8];
    // dBpi_s = e^{cs_end - cs_s} Lam x_s + sum_t K2[t][s] C~_t   (tile of s, n = tx + 16 jj); bv_s += B_s . Lam x_s
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) acc[i][jj] = 0.f;
    tile_mac<8>(acc, nN, P, Xs, 1, ldP, Lam, 1, ldP, ty, tx);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int s = ty + 16 * i;
      float bp = 0.f;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        if (jj >= nN) break;
        bp = fmaf(Bs[s * ldN + tx + 16 * jj], acc[i][jj], bp);
        acc[i][jj] *= eend[s];
      }
      for (int o = 8; o > 0; o >>= 1) bp += __shfl_xor_sync(0xffffffffu, bp, o);
      if (tx == 0 && s < L) atomicAdd(&bv[s], bp);
    }
    tile_mac<8>(acc, nN, L, S2, BL, 1, C, ldN, 1, ty, tx);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int s = ty + 16 * i;
      if (s >= L) continue;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        if (jj >= nN) break;
        float* o = &a.dbpi[((m0 + s) * d.k + j) * d.GN + (size_t)g * N + tx + 16 * jj];
        if (d.hpg == 1) *o = acc[i][jj];
        else atomicAdd(o, acc[i][jj]);
      }
    }
    // dC~_t += sum_{s <= t} K2[t][s] B_s
    tile_mac<8>(dC, nN, L, S2, 1, BL, Bs, ldN, 1, ty, tx);
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
  for (int i = 0; i < 4; ++i) {
    const int t = ty + 16 * i;
    if (t >= L) continue;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      if (jj >= nN) break;
      float* o = &a.dct[(m0 + t) * d.GN + (size_t)g * N + tx + 16 * jj];
      if (d.hpg == 1) *o = dC[i][jj];
      else atomicAdd(o, dC[i][jj]);
    }
  }
  if (tid < 32) {
    // dA_r = sum_{t >= r} q_t (a shuffle scan over the tokens in reverse order, two per lane);
    // d dt_r = dA_r A_h;  dA_h += sum_r dA_r dt_r
    const int lane = tid;
    if (lane == 0) q[L - 1] += expf(cs_end) * red[0] + red[1];
    __syncwarp();
    const int r0 = L - 1 - lane, r1 = L - 33 - lane;
    float v0 = r0 >= 0 ? q[r0] : 0.f, v1 = r1 >= 0 ? q[r1] : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u0 = __shfl_up_sync(0xffffffffu, v0, o), u1 = __shfl_up_sync(0xffffffffu, v1, o);
      if (lane >= o) { v0 += u0; v1 += u1; }
    }
    v1 += __shfl_sync(0xffffffffu, v0, 31);
    const float Ah = a.A[h];
    float part = 0.f;
    if (r0 >= 0) {
      const size_t o = (m0 + r0) * d.H + h;
      a.ddt[o] = v0 * Ah;
      part = v0 * a.dt[o];
    }
    if (r1 >= 0) {
      const size_t o = (m0 + r1) * d.H + h;
      a.ddt[o] = v1 * Ah;
      part = fmaf(v1, a.dt[o], part);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) atomicAdd(&a.dA[h], part);
  }
}

template <bool kD>
cudaError_t launch_states_tc(const BwdArgs& a, dim3 grid, size_t smt, cudaStream_t s) {
  const void* k = a.d.P == 64 ? (const void*)bwd_states_tc_kernel<kD, 64> : (const void*)bwd_states_tc_kernel<kD, 128>;
  const cudaError_t e = set_max_dynamic_smem(k, smt);
  if (e != cudaSuccess) return e;
  if (a.d.P == 64) bwd_states_tc_kernel<kD, 64><<<grid, 128, smt, s>>>(a);
  else bwd_states_tc_kernel<kD, 128><<<grid, 128, smt, s>>>(a);
  return cudaSuccess;
}

template <class S, int PJ>
cudaError_t launch_bwd_typed(const BwdArgs& a, cudaStream_t s) {
  const Dims& d = a.d;
  const dim3 grid(a.nc, d.H, d.Bsz);
  // fp16 streams with N = 128 and P in {64, 128}: the end states and adjoint sources on the tensor cores
  const bool tc_states = std::is_same<S, __half>::value && d.N == 128 && (d.P == 64 || d.P == 128);
  const size_t sm1 = (BL + (size_t)BL * d.N + (size_t)BL * d.P) * 4;
  const size_t smt = states_tc_smem(d.P);
  cudaError_t e;
  if (tc_states) {
    e = launch_states_tc<false>(a, grid, smt, s);
    if (e != cudaSuccess) return e;
  } else {
    e = set_max_dynamic_smem((const void*)bwd_fwd_chunk_kernel<S, PJ>, sm1);
    if (e != cudaSuccess) return e;
    bwd_fwd_chunk_kernel<S, PJ><<<grid, kBT, sm1, s>>>(a);
  }
  const dim3 pgrid(ceil_div(d.N * d.P, kBT), d.H, d.Bsz);
  bwd_fwd_pass_kernel<<<pgrid, kBT, 0, s>>>(a);
  if (tc_states) {
    e = launch_states_tc<true>(a, grid, smt, s);
    if (e != cudaSuccess) return e;
  } else {
    e = set_max_dynamic_smem((const void*)bwd_d_kernel<S, PJ>, sm1);
    if (e != cudaSuccess) return e;
    bwd_d_kernel<S, PJ><<<grid, kBT, sm1, s>>>(a);
  }
  bwd_adj_pass_kernel<<<pgrid, kBT, 0, s>>>(a);
  const size_t sm5 = GradSmem(d.N, d.P).total * 4;
  e = set_max_dynamic_smem((const void*)bwd_grad_kernel<S, PJ>, sm5);
  if (e != cudaSuccess) return e;
  bwd_grad_kernel<S, PJ><<<grid, kBT, sm5, s>>>(a);
  count_launches(5);
  return cudaGetLastError();
}

// P in {16, 32, 64, 128}: the column-group count of the register tiles as a template argument
template <class S>
cudaError_t launch_bwd_p(const BwdArgs& a, cudaStream_t s) {
  switch (a.d.P) {
    case 16: return launch_bwd_typed<S, 1>(a, s);
    case 32: return launch_bwd_typed<S, 2>(a, s);
    case 64: return launch_bwd_typed<S, 4>(a, s);
    case 128: return launch_bwd_typed<S, 8>(a, s);
    default: return cudaErrorInvalidValue;
  }
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
            hstart, work, cse, device_status()};
  if (!a.st) return cudaErrorInvalidValue;
  // the A gradient, and with G < H the Bpi and C~ gradients (summed over a group's heads), are accumulated
  cudaError_t e = cudaMemsetAsync(dA, 0, (size_t)d.H * 4, s);
  if (e == cudaSuccess && d.hpg > 1) e = cudaMemsetAsync(dbpi, 0, (size_t)d.M * d.k * d.GN * 4, s);
  if (e == cudaSuccess && d.hpg > 1) e = cudaMemsetAsync(dct, 0, (size_t)d.M * d.GN * 4, s);
  if (e != cudaSuccess) return e;
  return d.dtype == SWIMBA_BF16 ? launch_bwd_p<__half>(a, s) : launch_bwd_p<float>(a, s);
}

}  // namespace swimba
