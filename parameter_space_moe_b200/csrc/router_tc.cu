// Router and dt projection on the 5th-generation tensor cores (bf16 layers).
//
// Paper: Swimba notes, Method, flowchart node "token router R(X_t)" and key design 1 (pi_t = softmax(g_t)
// over the active set K_t); dt_t,h = clamp(softplus(W_dt[h] . X_t + b_dt[h]), 1e-3, 0.1).
// The E + H dot products of a token form one row of the skinny product X [M x D] . [W_r; W_dt]^T, whose
// cost is reading X once.  A 128-token tile is owned by a cluster of C CTAs (C in {1, 2, 4}) that split the
// K dimension, so that even a few thousand tokens spread the read of X over every SM.  In each CTA one
// thread streams its 64-wide K slices of X and of the stacked weights through a TMA ring (W_r rows at the
// top of the B tile, W_dt rows from row ceil8(E)) and issues tcgen05.mma M128 N=RP into TMEM (fp32).
// Each thread then reads its token row of partial logits from TMEM and stores it into the shared memory of
// the cluster CTA that finishes that token (token rows are dealt to the C CTAs in blocks of 128/C); after
// a cluster barrier each CTA sums the C partials in a fixed order, threads over (token, head) finish dt
// and one thread per token takes the top-k (k passes, strict '>' so equal logits keep the lower expert
// index) and counts its pairs per dispatch tile.
#include "tc_common.cuh"

namespace swimba {

namespace {
constexpr int RBM = 128, RBK = 64, kMaxStages = 12;
constexpr uint32_t kXStage = RBM * RBK * 2;  // 16 KB

struct RouterTcArgs {
  Dims d;
  int RP, eoff;  // padded logit columns, first dt column (ceil8(E))
  int stages;    // TMA ring depth
  int C;         // CTAs per token tile (cluster size, K split)
  const float* bdt;
  int32_t* idx;
  float* w;
  float* dt;
  int32_t* counts;
  unsigned* st;
};

// Shared-memory layout (offsets from the 1024-aligned base).
// With C == 1 the logits reuse the ring (written only after the last MMA completed); with C > 1 other CTAs
// store into them while this CTA's copies may still be landing, so they get their own region.
struct RouterSmem {
  uint32_t stage_bytes, ring, gs, g_off, bdt_off, bar_off, total;
  __host__ __device__ RouterSmem(int RP, int stages, int H, int C) {
    stage_bytes = kXStage + (uint32_t)RP * 128u;
    ring = (uint32_t)stages * stage_bytes;
    gs = (uint32_t)RP + 4u;  // partial-logit row stride in floats (16-byte aligned rows)
    const uint32_t g_bytes = (uint32_t)RBM * gs * 4u;
    g_off = C > 1 ? ring : 0u;
    const uint32_t end = C > 1 ? ring + g_bytes : (ring > g_bytes ? ring : g_bytes);
    bdt_off = end;
    bar_off = (bdt_off + (uint32_t)H * 4u + 7u) & ~7u;
    total = bar_off + (2 * kMaxStages + 1) * 8 + 8;
  }
};

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
      "[%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t e) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(e)
               : "memory");
}

__global__ void __launch_bounds__(128)
router_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wr,
                 const __grid_constant__ CUtensorMap tm_wdt, RouterTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const Dims& d = a.d;
  const int RP = a.RP, C = a.C;
  const RouterSmem L(RP, a.stages, d.H, C);
  float* G = reinterpret_cast<float*>(sm + L.g_off);  // [C sources][128 / C rows][gs] partial logits
  float* bdt_s = reinterpret_cast<float*>(sm + L.bdt_off);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bar_off);
  uint64_t* empty = full + kMaxStages;
  uint64_t* done = empty + kMaxStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  griddep_launch_dependents();  // the dispatch may start its prologue; it waits for this grid to finish
  const uint32_t rank = C > 1 ? tc::cluster_ctarank() : 0u;
  const int tile = blockIdx.x / C;
  const int tok0 = tile * RBM;
  const int R = RBM / C;                    // token rows this CTA finishes
  const int nkb = d.D / RBK / C;            // this CTA's K blocks
  const int kb0 = (int)rank * nkb;
  const uint32_t tx_bytes = kXStage + (uint32_t)(d.E + d.H) * 128u;
  const uint32_t idesc = tc::idesc_f16(RBM, RP, /*bf16=*/true);
  const uint32_t tcols = RP <= 32 ? 32u : (RP <= 64 ? 64u : 128u);
  volatile int never = 0;

  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s) { tc::mbar_init(&full[s], 1); tc::mbar_init(&empty[s], 1); }
    tc::mbar_init(done, 1);
    tc::fence_barrier_init();
  }
  for (int h = tid; h < d.H; h += 128) bdt_s[h] = a.bdt[h];
  if (warp == 0) { tc::tmem_alloc(tslot, tcols); tc::tmem_relinquish(); }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;
  // every CTA of the cluster has started (its shared memory exists) once this barrier phase completes;
  // waited for just before the first store into another CTA's shared memory
  if (C > 1) tc::cluster_arrive_relaxed();

  bool ok = true;
  if (tid == 0) {  // producer + MMA issuer; the rest of warp 0 waits at the __syncwarp below, not on `done`
    const int S = a.stages;
    int issued = 0;
    auto issue = [&](int kb) {
      const int s = kb % S;
      uint8_t* xs = sm + s * L.stage_bytes;
      uint8_t* ws = xs + kXStage;
      const int kc = (kb0 + kb) * RBK;
      tc::mbar_arrive_expect_tx(&full[s], tx_bytes);
      tc::tma_load_2d(xs, &tm_x, &full[s], kc, tok0);
      tc::tma_load_2d(ws, &tm_wr, &full[s], kc, 0);
      tc::tma_load_2d(ws + a.eoff * 128, &tm_wdt, &full[s], kc, 0);
      ++issued;
    };
    for (int kb = 0; kb < nkb && kb < S; ++kb) issue(kb);
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % S;
      if (!tc::mbar_wait(&full[s], (uint32_t)((kb / S) & 1), &never)) { ok = false; break; }
      tc::fence_after_sync();
      const uint32_t xa = tc::smem_u32(sm + s * L.stage_bytes), wa = xa + kXStage;
#pragma unroll
      for (int kk = 0; kk < RBK / 16; ++kk)
        tc::mma_f16(tmem, tc::sdesc_kmajor_sw128(xa + kk * 32), tc::sdesc_kmajor_sw128(wa + kk * 32), idesc,
                    (kb | kk) != 0);
      tc::mma_commit(&empty[s]);
      // refill the stage the previous k-block used once its MMAs are done (this block's MMAs keep the
      // tensor pipe busy meanwhile)
      const int r = kb - 1;
      if (r >= 0 && r + S < nkb) {
        if (!tc::mbar_wait(&empty[r % S], (uint32_t)((r / S) & 1), &never)) { ok = false; break; }
        issue(r + S);
      }
    }
    tc::mma_commit(done);
    if (!ok) {
      atomicOr(a.st, ST_TIMEOUT);
      // let the copies still in flight land before the CTA exits
      for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
        tc::mbar_wait(&full[i % S], (uint32_t)((i / S) & 1), &never);
    }
  }
  __syncwarp();
  ok = tc::mbar_wait(done, 0, &never) && ok;
  ok = __syncthreads_and(ok);
  tc::fence_after_sync();
  if (C > 1) tc::cluster_wait();
  {
    // this thread's token row (TMEM lane tid) of partial logits -> row (tid % R) of source slot `rank` in
    // the finishing CTA (tid / R)
    const uint32_t dst = tc::map_shared(tc::smem_u32(G) + ((rank * R + (tid % R)) * L.gs) * 4u, (uint32_t)(tid / R));
    if (ok) {
      for (int c = 0; c < RP; c += 16) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c, r);
        tc::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; e += 4) st_cluster_v4(dst + (c + e) * 4u, r[e], r[e + 1], r[e + 2], r[e + 3]);
      }
    }
  }
  tc::fence_before_sync();
  if (C > 1) tc::cluster_sync(); else __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, tcols);
  }
  ok = __syncthreads_and(ok);
  if (!ok) return;
  // The rest runs on 4 warps per CTA, so every loop below gives each thread kU independent items at a time
  // (loads first, then arithmetic, then stores) instead of one dependent chain per item.
  constexpr int kU = 8;
  // logits of this CTA's R tokens: sum of the C partials, source order 0 .. C-1 (float4 columns)
  if (C > 1) {
    const int q = RP / 4, n4 = R * q;
    for (int i0 = tid; i0 < n4; i0 += 128 * kU) {
      float4 acc[kU];
      int off[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i = i0 + u * 128;
        const int r = i / q, c4 = i - r * q;
        off[u] = r * (int)L.gs + 4 * c4;
        if (i < n4) acc[u] = *reinterpret_cast<const float4*>(G + off[u]);
      }
      for (int src = 1; src < C; ++src) {
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          if (i0 + u * 128 < n4) {
            const float4 v = *reinterpret_cast<const float4*>(G + src * R * (int)L.gs + off[u]);
            acc[u].x += v.x; acc[u].y += v.y; acc[u].z += v.z; acc[u].w += v.w;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (i0 + u * 128 < n4) *reinterpret_cast<float4*>(G + off[u]) = acc[u];
    }
    __syncthreads();
  }
  const int m0 = tok0 + (int)rank * R;  // first token this CTA finishes
  const int rows = min(R, d.M - m0);     // tokens of this CTA inside the batch
  for (int i0 = tid; i0 < rows * d.H; i0 += 128 * kU) {
    float v[kU];
    int r[kU], h[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * 128;
      r[u] = i / d.H;
      h[u] = i - r[u] * d.H;
      v[u] = i < rows * d.H ? G[r[u] * L.gs + a.eoff + h[u]] + bdt_s[h[u]] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const float sp = v[u] > 20.f ? v[u] : log1pf(expf(v[u]));
      if (i0 + u * 128 < rows * d.H) a.dt[(size_t)(m0 + r[u]) * d.H + h[u]] = fminf(fmaxf(sp, 1e-3f), 0.1f);
    }
  }
  // the counts table was cleared by the kernel before this one (launched with programmatic dependent launch
  // after it, this grid may have started early); without that launch mode the wait returns at once
  griddep_wait();
  if (tid < rows) {
    const int m = m0 + tid;
    const float* gl = G + tid * L.gs;
    unsigned long long taken = 0ull;
    float gsel[8];
    int isel[8];
    for (int j = 0; j < d.k; ++j) {
      int bi = -1;
      float bv = -INFINITY;
      for (int e0 = 0; e0 < d.E; e0 += 4) {
        const float4 g4 = *reinterpret_cast<const float4*>(gl + e0);  // E <= eoff, columns up to eoff exist
        const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = e0 + u;
          if (e < d.E && !((taken >> e) & 1ull) && (bi < 0 || gv[u] > bv)) { bv = gv[u]; bi = e; }
        }
      }
      taken |= 1ull << bi;
      gsel[j] = bv;
      isel[j] = bi;
    }
    float den = 0.f, ex[8];
    for (int j = 0; j < d.k; ++j) { ex[j] = expf(gsel[j] - gsel[0]); den += ex[j]; }
    for (int j = 0; j < d.k; ++j) {
      a.idx[(size_t)m * d.k + j] = isel[j];
      a.w[(size_t)m * d.k + j] = ex[j] / den;
      if (a.counts) atomicAdd(&a.counts[(size_t)((m * d.k + j) / kDispatchTile) * d.E + isel[j]], 1);
    }
  }
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) ==
                                                   cudaSuccess)
      n = v;
    else
      return 148;
  }
  return n;
}
}  // namespace

// bf16 layers whose padded logit row (ceil8(E) + H columns, rounded to 16) fits one M128 x N<=128 MMA.
bool router_tc_supported(const Dims& d) {
  const int eoff = (d.E + 7) / 8 * 8;
  return d.dtype == SWIMBA_BF16 && d.D % RBK == 0 && eoff + d.H <= 128;
}

// Returns cudaErrorNotSupported, with nothing launched, when a tensor map cannot be encoded (the caller
// then takes another router kernel).
cudaError_t launch_router_tc(const Dims& d, const void* X, const swimba_weights& w, int32_t* idx, float* wts,
                             float* dt, int32_t* counts, unsigned* st, cudaStream_t s, bool after_zero) {
  const int eoff = (d.E + 7) / 8 * 8;
  const int RP = (eoff + d.H + 15) / 16 * 16;
  CUtensorMap tx, twr, twd;
  if (!encode_tmap_2d(&tx, X, SWIMBA_BF16, (uint64_t)d.D, (uint64_t)d.M, (uint64_t)d.D * 2, RBK, RBM) ||
      !encode_tmap_2d(&twr, w.w_router, SWIMBA_BF16, (uint64_t)d.D, (uint64_t)d.E, (uint64_t)d.D * 2, RBK, d.E) ||
      !encode_tmap_2d(&twd, w.w_dt, SWIMBA_BF16, (uint64_t)d.D, (uint64_t)d.H, (uint64_t)d.D * 2, RBK, d.H))
    return cudaErrorNotSupported;
  // K split: double the cluster while the grid has fewer CTAs than SMs and the K blocks divide evenly.
  const int nblk = ceil_div(d.M, RBM), nkb = d.D / RBK, nsm = sm_count();
  int C = 1;
  while (C < 4 && nblk * C < nsm && nkb % (2 * C) == 0) C *= 2;
  // Ring depth: up to ~80 KB of copies in flight per CTA (two CTAs share an SM), at most the CTA's K blocks.
  const size_t stage_bytes = kXStage + (size_t)RP * 128;
  int S = (int)((80u << 10) / stage_bytes);
  S = S < 2 ? 2 : (S > kMaxStages ? kMaxStages : S);
  if (S > nkb / C) S = nkb / C;
  const RouterSmem L(RP, S, d.H, C);
  const size_t smem = 1024 + L.total;
  RouterTcArgs a{d, RP, eoff, S, C, w.b_dt, idx, wts, dt, counts, st};
  cudaError_t e = set_max_dynamic_smem((const void*)router_tc_kernel, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nblk * C));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_zero ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, router_tc_kernel, tx, twr, twd, a);
  count_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace swimba
