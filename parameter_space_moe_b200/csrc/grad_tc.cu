// Gradients of the expert projections on the 5th-generation tensor cores (bf16 layers):
//   dXp[p]   = dz[p] W_e                              for every (token, slot) pair p routed to expert e
//   dW_e     = sum over the pairs p routed to e of dz[p]^T X[token(p)]
// where z = [x | B | C] is expert e's projection of X[token(p)] and dz its gradient.
//
// Paper: Swimba notes, key design 1 (each active expert projects X_t into its candidate streams) and the
// training section (the layer is trained end to end, so the projection weights and X receive gradients);
// the products above are the reverse mode of the forward's Z = X W_e^T.
//
// dz is fp32.  Each product runs on a bf16 split dz = hi + lo (hi = bf16(dz), lo = bf16(dz - hi)): two
// bf16 MMAs into one fp32 TMEM accumulator, so the operand rounding stays near 2^-17 relative -- the same
// accuracy class as fp32 CUDA-core arithmetic -- while X and W_e are exact in bf16.
//
// Operands, in "padded sorted" row order rp (expert e's sorted rows start at poff[e], a multiple of 64, and
// its segment is padded with zero rows up to the next multiple of 64); the pack kernel below lays out the rows
// and the mix gradient writes each pair's dz split into its padded row:
//   dzs [Rp][2 Wp] bf16   row rp = [hi(dz) | 0 | lo(dz) | 0] of the pair there (Wp = W_e rounded up to 64)
//   xsp [Rp][D]    bf16   X row of that pair's token, zero on pad rows
//   prow[Rp]       int32  the pair index, -1 on pad rows
// dX product: A = dzs (K-major, K = 2 Wp), B = W_e [W_e][D] read MN-major (N = D) -- no transposed copy.
// dW product: A = dzs read MN-major (M = W_e columns, K = the expert's padded rows), B = xsp MN-major.
// Both use 128 x 256 tiles, 64-deep K stages, fp32 accumulators double-buffered in TMEM (512 columns),
// one persistent CTA per SM: warp 0 TMA producer, warp 1 TMEM owner and MMA issuer, warps 2..9 epilogue.
#include "tc_common.cuh"

namespace swimba {

namespace {
constexpr int BM = 128, BN = 256, BK = 64, kStages = 4;
constexpr int kEpiWarps = 8;  // 2 per TMEM lane quarter, each draining 128 of the 256 columns
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kStageA = BM * BK * 2, kStageB = BN * BK * 2, kStageBytes = kStageA + kStageB;
constexpr uint32_t kBlk = 64 * 128;  // one MN-major block: 64 K rows of 128 bytes (64 MN values)
constexpr uint32_t kTmemCols = 2 * BN;
constexpr uint32_t kIdescDx = tc::idesc_f16(BM, BN, /*bf16=*/true, /*a_mn=*/false, /*b_mn=*/true);
constexpr uint32_t kIdescDw = tc::idesc_f16(BM, BN, /*bf16=*/true, /*a_mn=*/true, /*b_mn=*/true);
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 1024;
constexpr int kMaxE = 64;

struct GArgs {
  int kind;  // 0: dX product, 1: dW product
  int E, We, Wp, D;
  const int32_t* poff;  // [E+1] padded expert offsets
  const int32_t* offsets;  // [E+1] expert offsets in sorted rows
  const int32_t* prow;  // [Rp] pair index per padded row, -1 on pad rows
  float* out;           // kind 0: dXp [M*k][D]; kind 1: dW_exp [E][W_e][D]
  unsigned* st;
};

// Tile t: its expert, its K blocks (half of them on the hi part of dz, then as many on the lo part), and its
// first output row (padded sorted row, or W_e column) and column.
struct Tile {
  int e, nkb, half;
  int m0, n0;
};

__device__ __forceinline__ bool resolve(const GArgs& g, const int* poff_s, const int* tpre_s, int t, Tile& T) {
  const int nct = ceil_div(g.D, BN);
  if (g.kind == 0) {
    const int rt = t / nct;
    if (rt >= tpre_s[g.E]) return false;
    int e = 0;
    while (e + 1 < g.E && tpre_s[e + 1] <= rt) ++e;
    T.e = e;
    T.m0 = poff_s[e] + (rt - tpre_s[e]) * BM;
    T.n0 = (t % nct) * BN;
    T.half = g.Wp / BK;
    T.nkb = 2 * T.half;
  } else {
    const int mct = ceil_div(g.We, BM);
    T.e = t / (mct * nct);
    if (T.e >= g.E) return false;
    const int rem = t % (mct * nct);
    T.m0 = (rem / nct) * BM;
    T.n0 = (rem % nct) * BN;
    T.half = (poff_s[T.e + 1] - poff_s[T.e]) / BK;
    T.nkb = 2 * T.half;
  }
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
grad_tc_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b, GArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = bars + 2 * kStages + 2;
  uint64_t* drain = bars + 2 * kStages + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ int poff_s[kMaxE + 1], tpre_s[kMaxE + 1], off_s[kMaxE + 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { tc::mbar_init(&full[s], 1); tc::mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&acc_full[b], 1); tc::mbar_init(&acc_empty[b], 32 * kEpiWarps); }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tmap_a);
    tc::tma_prefetch_desc(&tmap_b);
    // padded offsets and the prefix count of 128-row tiles per expert (dX product)
    int acc = 0;
    for (int e = 0; e <= g.E; ++e) {
      poff_s[e] = g.poff[e];
      off_s[e] = g.offsets[e];
      tpre_s[e] = acc;
      if (e < g.E) acc += ceil_div(g.poff[e + 1] - g.poff[e], BM);
    }
  }
  if (warp == 1) { tc::tmem_alloc(tmem_slot, kTmemCols); tc::tmem_relinquish(); }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    bool ok = true;
    Tile T;
    for (int t = blockIdx.x; ok && resolve(g, poff_s, tpre_s, t, T); t += gridDim.x) {
      for (int kb = 0; kb < T.nkb; ++kb) {
        if (!tc::mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        uint8_t* sa = stage_base + stage * kStageBytes;
        uint8_t* sb = sa + kStageA;
        tc::mbar_arrive_expect_tx(&full[stage], kStageBytes);
        const bool lo = kb >= T.half;
        const int kq = (lo ? kb - T.half : kb) * BK;
        if (g.kind == 0) {
          // A: dzs rows m0.., columns kb*64 (hi blocks then lo blocks); B: W_e rows e*We + kq, 4 x 64 columns
          tc::tma_load_2d(sa, &tmap_a, &full[stage], kb * BK, T.m0);
          for (int j = 0; j < 4; ++j)
            tc::tma_load_2d(sb + j * kBlk, &tmap_b, &full[stage], T.n0 + 64 * j, T.e * g.We + kq);
        } else {
          // A: dzs rows poff[e] + kq, W_e columns m0.. (+ Wp for the lo part); B: xsp rows poff[e] + kq
          const int r = poff_s[T.e] + kq;
          for (int j = 0; j < 2; ++j)
            tc::tma_load_2d(sa + j * kBlk, &tmap_a, &full[stage], T.m0 + 64 * j + (lo ? g.Wp : 0), r);
          for (int j = 0; j < 4; ++j) tc::tma_load_2d(sb + j * kBlk, &tmap_b, &full[stage], T.n0 + 64 * j, r);
        }
        ++issued;
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok) { *abort_flag = 1; atomicOr(g.st, ST_TIMEOUT); }
    for (long long i = 0; i < kStages && i < issued; ++i) {
      if (--stage < 0) { stage = kStages - 1; phase ^= 1u; }
      volatile int never = 0;
      tc::mbar_wait(&full[stage], phase, &never);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int buf = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    Tile T;
    for (int t = blockIdx.x; ok && resolve(g, poff_s, tpre_s, t, T); t += gridDim.x) {
      if (!tc::mbar_wait(&acc_empty[buf], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
      tc::fence_after_sync();
      const uint32_t dt = tmem + (uint32_t)(buf * BN);
      for (int kb = 0; kb < T.nkb; ++kb) {
        if (!tc::mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t sa = tc::smem_u32(stage_base + stage * kStageBytes), sb = sa + kStageA;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          // MN-major operands step 16 K rows = 2048 bytes; the K-major A steps 32 bytes inside its rows
          const uint64_t db = tc::sdesc_mnmajor_sw128(sb + kk * 2048, kBlk);
          if (g.kind == 0)
            tc::mma_f16(dt, tc::sdesc_kmajor_sw128(sa) + 2 * kk, db, kIdescDx, (kb | kk) != 0);
          else
            tc::mma_f16(dt, tc::sdesc_mnmajor_sw128(sa + kk * 2048, kBlk), db, kIdescDw, (kb | kk) != 0);
        }
        tc::mma_commit(&empty[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      tc::mma_commit(&acc_full[buf]);
      if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
    }
    if (!ok) { *abort_flag = 1; atomicOr(g.st, ST_TIMEOUT); }
    tc::mma_commit(drain);
    volatile int never = 0;
    tc::mbar_wait(drain, 0, &never);
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue: fp32 rows straight to HBM
    const int q = warp & 3, part = (warp - 2) >> 2;
    const int rl = 32 * q + lane;
    int buf = 0;
    uint32_t acc_phase = 0;
    Tile T;
    for (int t = blockIdx.x; resolve(g, poff_s, tpre_s, t, T); t += gridDim.x) {
      float* dst = nullptr;
      if (g.kind == 0) {
        const int rp = T.m0 + rl;
        const int p = rp < poff_s[T.e] + (off_s[T.e + 1] - off_s[T.e]) ? g.prow[rp] : -1;
        if (p >= 0) dst = g.out + (size_t)p * g.D;
      } else if (T.m0 + rl < g.We) {
        dst = g.out + ((size_t)T.e * g.We + T.m0 + rl) * g.D;
      }
      if (!tc::mbar_wait(&acc_full[buf], acc_phase, abort_flag)) {
        *abort_flag = 1;
        atomicOr(g.st, ST_TIMEOUT);
        break;
      }
      tc::fence_after_sync();
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN + 128 * part);
      uint32_t ra[32], rb[32];
      tc::tmem_ld_32x32b_x32(taddr, ra);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t(&cur)[32] = (c & 1) ? rb : ra;
        uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
        tc::tmem_ld_wait(cur);
        if (c + 1 < 4) tc::tmem_ld_32x32b_x32(taddr + 32 * (c + 1), nxt);
        const int col = T.n0 + 128 * part + 32 * c;
        if (dst && col < g.D) {
          float* o = dst + col;
          const bool zero = T.nkb == 0;  // an expert with no rows: its weight gradient is 0
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(o + i) =
                zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                     : make_float4(__uint_as_float(cur[i]), __uint_as_float(cur[i + 1]),
                                   __uint_as_float(cur[i + 2]), __uint_as_float(cur[i + 3]));
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&acc_empty[buf]);
      if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// poff[e] = sum over experts e' < e of their row counts rounded up to 64 (one thread; E <= 64).
__global__ void pad_offsets_kernel(int E, const int32_t* __restrict__ offsets, int32_t* __restrict__ poff) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int acc = 0;
  for (int e = 0; e < E; ++e) {
    poff[e] = acc;
    acc += (offsets[e + 1] - offsets[e] + BK - 1) / BK * BK;
  }
  poff[E] = acc;
}

// One CTA per padded row rp: the row's pair (or -1), the pair's padded row (for the mix gradient, which writes
// the pair's dz split there), and the token's X row; a pad row's dz split is zeroed here.
template <class T>
__global__ void __launch_bounds__(256)
pack_rows_kernel(int E, int Wp, int D, const int32_t* __restrict__ poff, const int32_t* __restrict__ offsets,
                 const int32_t* __restrict__ perm, const T* __restrict__ xsorted, __nv_bfloat16* __restrict__ dzs,
                 __nv_bfloat16* __restrict__ xsp, int32_t* __restrict__ prow, int32_t* __restrict__ rp_of_p) {
  __shared__ int s_r;
  const int rp = blockIdx.x;
  if (threadIdx.x == 0) {
    int r = -1;
    if (rp < poff[E]) {
      int e = 0;
      while (e + 1 < E && poff[e + 1] <= rp) ++e;
      const int rr = offsets[e] + (rp - poff[e]);
      if (rr < offsets[e + 1]) r = rr;
    }
    s_r = r;
    const int p = r >= 0 ? perm[r] : -1;
    prow[rp] = p;
    if (p >= 0) rp_of_p[p] = rp;
  }
  __syncthreads();
  const int r = s_r;
  if (r < 0) {
    uint2* z = reinterpret_cast<uint2*>(dzs + (size_t)rp * 2 * Wp);
    for (int c = threadIdx.x; c < Wp / 2; c += blockDim.x) z[c] = make_uint2(0u, 0u);
  }
  const T* xr = r >= 0 ? xsorted + (size_t)r * D : nullptr;
  for (int c = 4 * threadIdx.x; c < D; c += 4 * blockDim.x) {
    uint2 u = make_uint2(0u, 0u);
    if (xr) u = *reinterpret_cast<const uint2*>(xr + c);
    *reinterpret_cast<uint2*>(xsp + (size_t)rp * D + c) = u;
  }
}

int sm_count() {
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}
}  // namespace

size_t grad_tc_rows(const Dims& d) { return align_up((size_t)d.M * d.k + (size_t)64 * d.E, 128); }
int grad_tc_wp(const Dims& d) { return ceil_div(d.We, BK) * BK; }

// The operand layout of the expert products: padded offsets, pair per padded row and padded row per pair,
// padded X rows, zeroed pad rows of the dz split (the mix gradient fills the others).  bf16 layers only.
cudaError_t launch_grad_tc_pack(const Dims& d, const void* xsorted, const int32_t* perm, const int32_t* offsets,
                                int32_t* poff, int32_t* prow, int32_t* rp_of_p, void* dzs, void* xsp, cudaStream_t s) {
  if (d.dtype != SWIMBA_BF16 || d.E > kMaxE) return cudaErrorInvalidValue;
  const int Rp = (int)grad_tc_rows(d), Wp = grad_tc_wp(d);
  pad_offsets_kernel<<<1, 32, 0, s>>>(d.E, offsets, poff);
  pack_rows_kernel<__nv_bfloat16><<<Rp, 256, 0, s>>>(d.E, Wp, d.D, poff, offsets, perm,
                                                      (const __nv_bfloat16*)xsorted, (__nv_bfloat16*)dzs,
                                                      (__nv_bfloat16*)xsp, prow, rp_of_p);
  count_launches(2);
  return cudaGetLastError();
}

// dXp (per pair) and dW_exp from the packed operands.
cudaError_t launch_grad_tc(const Dims& d, const void* w_exp, const int32_t* offsets, const int32_t* poff,
                           const int32_t* prow, const void* dzs, const void* xsp, float* dxp, float* dW_exp,
                           unsigned* st, cudaStream_t s) {
  if (d.dtype != SWIMBA_BF16 || d.E > kMaxE) return cudaErrorInvalidValue;
  const int Rp = (int)grad_tc_rows(d), Wp = grad_tc_wp(d);
  CUtensorMap ta_dx, ta_dw, tb_dx, tb_dw;
  if (!encode_tmap_2d(&ta_dx, dzs, SWIMBA_BF16, (uint64_t)2 * Wp, (uint64_t)Rp, (uint64_t)2 * Wp * 2, BK, BM) ||
      !encode_tmap_2d(&ta_dw, dzs, SWIMBA_BF16, (uint64_t)2 * Wp, (uint64_t)Rp, (uint64_t)2 * Wp * 2, 64, BK) ||
      !encode_tmap_2d(&tb_dx, w_exp, SWIMBA_BF16, (uint64_t)d.D, (uint64_t)d.E * d.We, (uint64_t)d.D * 2, 64, BK) ||
      !encode_tmap_2d(&tb_dw, xsp, SWIMBA_BF16, (uint64_t)d.D, (uint64_t)Rp, (uint64_t)d.D * 2, 64, BK))
    return cudaErrorInvalidValue;
  cudaError_t e = set_max_dynamic_smem((const void*)grad_tc_kernel, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int sms = sm_count();
  GArgs g{0, d.E, d.We, Wp, d.D, poff, offsets, prow, dxp, st};
  const int dx_tiles = (Rp / BM + d.E) * ceil_div(d.D, BN);
  grad_tc_kernel<<<dx_tiles < sms ? dx_tiles : sms, kThreads, kSmemBytes, s>>>(ta_dx, tb_dx, g);
  g.kind = 1;
  g.out = dW_exp;
  const int dw_tiles = d.E * ceil_div(d.We, BM) * ceil_div(d.D, BN);
  grad_tc_kernel<<<dw_tiles < sms ? dw_tiles : sms, kThreads, kSmemBytes, s>>>(ta_dw, tb_dw, g);
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace swimba
