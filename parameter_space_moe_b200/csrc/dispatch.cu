// Expert dispatch: a stable counting sort of the M*k (token, slot) pairs by expert, plus the row-tile
// schedule of the grouped expert GEMM and the gather of X rows into expert-major order.
//
// Pair p = m*k + j (token m, slot j) has expert topk_idx[p].  Standalone dispatch (swimba_dispatch,
// swimba_expert_proj), three launches:
//   count    one CTA per tile of kDispatchTile consecutive pairs: per-expert counts of the tile
//   offsets  one CTA: expert_offsets (exclusive prefix of the totals), each (tile, expert)'s first
//            sorted position, and the GEMM schedule (expert, first row) of kRowTile-row tiles
//   scatter  one CTA per tile: stable rank of each pair inside its tile (warp match + per-warp
//            prefix), perm[position] = p
// Inside the layer the router already produced the per-tile counts, so one launch does the rest:
// dispatch_fused_kernel (fp32 layers, followed by no gather) or dispatch_gather_kernel (bf16 layers,
// which also copies the X rows into expert order for the tensor-core GEMM).
// The order inside an expert is increasing p, so the permutation is deterministic.
#include "common.cuh"

namespace swimba {

constexpr int kDispatchThreads = 1024;

// Caller-given indices outside [0, E) are skipped (and reported through the status word) so that no
// shared-memory table is indexed out of bounds.
__global__ void __launch_bounds__(kDispatchThreads)
dispatch_count_kernel(Dims d, const int32_t* __restrict__ idx, int32_t* __restrict__ counts, unsigned* st) {
  __shared__ int c_s[64];
  const int tile = blockIdx.x;
  if (threadIdx.x < 64) c_s[threadIdx.x] = 0;
  __syncthreads();
  const int total = d.M * d.k;
  bool bad = false;
  for (int i = threadIdx.x; i < kDispatchTile; i += blockDim.x) {
    int p = tile * kDispatchTile + i;
    if (p < total) {
      const int e = idx[p];
      if (e >= 0 && e < d.E) atomicAdd(&c_s[e], 1);
      else bad = true;
    }
  }
  if (bad) atomicOr(st, ST_INDEX);
  __syncthreads();
  if (threadIdx.x < d.E) counts[tile * d.E + threadIdx.x] = c_s[threadIdx.x];
}

__global__ void __launch_bounds__(1024)
dispatch_offsets_kernel(Dims d, int ntile, const int32_t* __restrict__ counts, int32_t* __restrict__ base,
                        int32_t* __restrict__ offsets, int32_t* __restrict__ tiles, int32_t* __restrict__ ntiles) {
  __shared__ int tot_s[65];
  __shared__ int off_s[65];
  __shared__ int toff_s[65];
  const int e = threadIdx.x;
  if (e < d.E) {
    int t = 0;
    for (int i = 0; i < ntile; ++i) t += counts[i * d.E + e];
    tot_s[e] = t;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int o = 0, to = 0;
    for (int x = 0; x < d.E; ++x) {
      off_s[x] = o; toff_s[x] = to;
      o += tot_s[x]; to += ceil_div(tot_s[x], kRowTile);
    }
    off_s[d.E] = o; toff_s[d.E] = to;
    *ntiles = to;
  }
  __syncthreads();
  if (e <= d.E) offsets[e] = off_s[e];
  if (e < d.E) {
    int o = off_s[e];
    for (int i = 0; i < ntile; ++i) { base[i * d.E + e] = o; o += counts[i * d.E + e]; }
  }
  // GEMM schedule: tile r of expert e covers sorted rows [off + r*kRowTile, min(off_{e+1}, ...))
  for (int x = 0; x < d.E; ++x) {
    const int nt = ceil_div(tot_s[x], kRowTile);
    for (int r = threadIdx.x; r < nt; r += blockDim.x) {
      tiles[2 * (toff_s[x] + r) + 0] = x;
      tiles[2 * (toff_s[x] + r) + 1] = off_s[x] + r * kRowTile;
    }
  }
}

__global__ void __launch_bounds__(kDispatchThreads)
dispatch_scatter_kernel(Dims d, const int32_t* __restrict__ idx, const int32_t* __restrict__ base,
                        int32_t* __restrict__ perm, int2* __restrict__ rowmeta, const float* __restrict__ topk_w) {
  __shared__ int wc_s[kDispatchThreads / 32][64];  // per-warp counts, turned into per-warp bases
  const int tile = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = d.M * d.k;
  for (int x = threadIdx.x; x < (kDispatchThreads / 32) * 64; x += blockDim.x) (&wc_s[0][0])[x] = 0;
  __syncthreads();
  const int p = tile * kDispatchTile + threadIdx.x;  // kDispatchTile == blockDim.x
  const int raw = p < total ? idx[p] : 0;
  const bool valid = p < total && raw >= 0 && raw < d.E;  // out-of-range indices were reported by the count
  const int e = valid ? raw : -1 - lane;             // distinct sentinels never match a real expert
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (valid && rank == 0) wc_s[warp][e] = __popc(peers);
  __syncthreads();
  if (threadIdx.x < d.E) {
    int run = base[tile * d.E + threadIdx.x];
    for (int w = 0; w < kDispatchThreads / 32; ++w) {
      int c = wc_s[w][threadIdx.x];
      wc_s[w][threadIdx.x] = run;
      run += c;
    }
  }
  __syncthreads();
  if (valid) {
    const int pos = wc_s[warp][e] + rank;
    perm[pos] = p;
    if (rowmeta) rowmeta[pos] = make_int2(p, topk_w ? __float_as_int(topk_w[p]) : 0);
  }
}

// The layer's dispatch in one launch: per-tile counts arrive from the router (integer atomics into a
// zeroed [tile][E] table), so each CTA derives the global expert offsets and its tile's bases itself
// (sums over at most M*k/1024 tiles), CTA 0 publishes expert_offsets and the GEMM row-tile schedule, and
// every CTA scatters its pairs with the same stable ranking as dispatch_scatter_kernel.
__global__ void __launch_bounds__(kDispatchThreads)
dispatch_fused_kernel(Dims d, const int32_t* __restrict__ idx, const int32_t* __restrict__ counts,
                      int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ tiles,
                      int32_t* __restrict__ ntiles, int2* __restrict__ rowmeta, const float* __restrict__ topk_w) {
  __shared__ int wc_s[kDispatchThreads / 32][64];
  __shared__ int tot_s[64], pre_s[64], off_s[65], toff_s[65];
  const int tile = blockIdx.x, ntile = gridDim.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = d.M * d.k;
  griddep_launch_dependents();
  griddep_wait();  // the router's counts, indices and weights
  if (threadIdx.x < d.E) {
    const int e = threadIdx.x;
    int t = 0, pre = 0;
    for (int i = 0; i < ntile; ++i) {
      const int c = counts[i * d.E + e];
      t += c;
      if (i < tile) pre += c;
    }
    tot_s[e] = t;
    pre_s[e] = pre;
  }
  for (int x = threadIdx.x; x < (kDispatchThreads / 32) * 64; x += blockDim.x) (&wc_s[0][0])[x] = 0;
  __syncthreads();
  if (threadIdx.x == 0) {
    int o = 0, to = 0;
    for (int e = 0; e < d.E; ++e) {
      off_s[e] = o; toff_s[e] = to;
      o += tot_s[e]; to += ceil_div(tot_s[e], kRowTile);
    }
    off_s[d.E] = o; toff_s[d.E] = to;
    if (tile == 0) *ntiles = to;
  }
  __syncthreads();
  if (tile == 0) {
    if (threadIdx.x <= d.E) offsets[threadIdx.x] = off_s[threadIdx.x];
    for (int e = 0; e < d.E; ++e) {
      const int nt = ceil_div(tot_s[e], kRowTile);
      for (int r = threadIdx.x; r < nt; r += blockDim.x) {
        tiles[2 * (toff_s[e] + r) + 0] = e;
        tiles[2 * (toff_s[e] + r) + 1] = off_s[e] + r * kRowTile;
      }
    }
  }
  const int p = tile * kDispatchTile + threadIdx.x;
  const bool valid = p < total;
  const int e = valid ? idx[p] : -1 - lane;
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (valid && rank == 0) wc_s[warp][e] = __popc(peers);
  __syncthreads();
  if (threadIdx.x < d.E) {
    int run = off_s[threadIdx.x] + pre_s[threadIdx.x];
    for (int w = 0; w < kDispatchThreads / 32; ++w) {
      const int c = wc_s[w][threadIdx.x];
      wc_s[w][threadIdx.x] = run;
      run += c;
    }
  }
  __syncthreads();
  if (valid) {
    const int pos = wc_s[warp][e] + rank;
    perm[pos] = p;
    rowmeta[pos] = make_int2(p, __float_as_int(topk_w[p]));
  }
}

// The layer's dispatch with the row gather fused in: `split` CTAs per dispatch tile each rank the whole
// tile (cheap: one match per warp and a per-expert running sum over the warps) and then copy the X rows
// of their own kDispatchTile / split pairs into expert-major order, so the gather's bytes are spread over
// enough CTAs to draw HBM bandwidth and the separate gather launch disappears.
constexpr int kMaxPartPairs = kDispatchTile / 8;  // at least 8 CTAs per tile
template <class T>
__global__ void __launch_bounds__(kDispatchThreads)
dispatch_gather_kernel(Dims d, const int32_t* __restrict__ idx, const int32_t* __restrict__ counts,
                       int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ tiles,
                       int32_t* __restrict__ ntiles, int2* __restrict__ rowmeta, const float* __restrict__ topk_w,
                       const T* __restrict__ X, T* __restrict__ xs, int split) {
  __shared__ int wc_s[kDispatchThreads / 32][64];
  __shared__ int tot_s[64], pre_s[64], off_s[65], toff_s[65];
  __shared__ int pos_s[kMaxPartPairs];
  const int tile = blockIdx.x / split, part = blockIdx.x % split, ntile = gridDim.x / split;
  const int part_pairs = kDispatchTile / split;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = d.M * d.k;
  griddep_launch_dependents();
  griddep_wait();  // the router's counts, indices and weights
  if (threadIdx.x < d.E) {
    const int e = threadIdx.x;
    int t = 0, pre = 0;
    for (int i = 0; i < ntile; ++i) {
      const int c = counts[i * d.E + e];
      t += c;
      if (i < tile) pre += c;
    }
    tot_s[e] = t;
    pre_s[e] = pre;
  }
  for (int x = threadIdx.x; x < (kDispatchThreads / 32) * 64; x += blockDim.x) (&wc_s[0][0])[x] = 0;
  __syncthreads();
  if (threadIdx.x == 0) {
    int o = 0, to = 0;
    for (int e = 0; e < d.E; ++e) {
      off_s[e] = o; toff_s[e] = to;
      o += tot_s[e]; to += ceil_div(tot_s[e], kRowTile);
    }
    off_s[d.E] = o; toff_s[d.E] = to;
    if (blockIdx.x == 0) *ntiles = to;
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    if (threadIdx.x <= d.E) offsets[threadIdx.x] = off_s[threadIdx.x];
    for (int e = 0; e < d.E; ++e) {
      const int nt = ceil_div(tot_s[e], kRowTile);
      for (int r = threadIdx.x; r < nt; r += blockDim.x) {
        tiles[2 * (toff_s[e] + r) + 0] = e;
        tiles[2 * (toff_s[e] + r) + 1] = off_s[e] + r * kRowTile;
      }
    }
  }
  const int p = tile * kDispatchTile + threadIdx.x;
  const bool valid = p < total;
  const int e = valid ? idx[p] : -1 - lane;
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (valid && rank == 0) wc_s[warp][e] = __popc(peers);
  __syncthreads();
  if (threadIdx.x < d.E) {
    int run = off_s[threadIdx.x] + pre_s[threadIdx.x];
    for (int w = 0; w < kDispatchThreads / 32; ++w) {
      const int c = wc_s[w][threadIdx.x];
      wc_s[w][threadIdx.x] = run;
      run += c;
    }
  }
  __syncthreads();
  if (valid && threadIdx.x / part_pairs == part) {
    const int pos = wc_s[warp][e] + rank;
    perm[pos] = p;
    rowmeta[pos] = make_int2(p, __float_as_int(topk_w[p]));
    pos_s[threadIdx.x % part_pairs] = pos;
  }
  __syncthreads();
  // this CTA's rows, one warp per row, 16-byte vectors, up to 8 loads in flight per lane
  const int nv = d.D * (int)sizeof(T) / 16;
  for (int r = warp; r < part_pairs; r += kDispatchThreads / 32) {
    const int pp = tile * kDispatchTile + part * part_pairs + r;
    if (pp >= total) break;
    const int4* src = reinterpret_cast<const int4*>(X + (size_t)(pp / d.k) * d.D);
    int4* dst = reinterpret_cast<int4*>(xs + (size_t)pos_s[r] * d.D);
    for (int i0 = 0; i0 < nv; i0 += 32 * 8) {
      int4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (i0 + lane + 32 * u < nv) v[u] = __ldg(src + i0 + lane + 32 * u);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (i0 + lane + 32 * u < nv) dst[i0 + lane + 32 * u] = v[u];
    }
  }
}

// X rows in sorted order: xsorted[r] = X[perm[r] / k].  One warp per row, 16-byte vectors.
template <class T>
__global__ void gather_rows_kernel(Dims d, const T* __restrict__ X, const int32_t* __restrict__ perm,
                                   T* __restrict__ xs) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  griddep_launch_dependents();
  griddep_wait();  // the dispatch's permutation
  if (warp >= d.M * d.k) return;
  const int m = perm[warp] / d.k;
  const int4* src = reinterpret_cast<const int4*>(X + (size_t)m * d.D);
  int4* dst = reinterpret_cast<int4*>(xs + (size_t)warp * d.D);
  const int nv = d.D * (int)sizeof(T) / 16;
  for (int i = lane; i < nv; i += 32) dst[i] = src[i];
}

cudaError_t launch_dispatch(const Dims& d, const int32_t* idx, const WsPlan& p, char* ws, int32_t* offsets,
                            int32_t* perm, int2* rowmeta, const float* topk_w, unsigned* st, cudaStream_t s) {
  const int nt = dispatch_tiles(d);
  int32_t* counts = (int32_t*)(ws + p.dcounts);
  int32_t* base = (int32_t*)(ws + p.dbase);
  dispatch_count_kernel<<<nt, kDispatchThreads, 0, s>>>(d, idx, counts, st);
  dispatch_offsets_kernel<<<1, 1024, 0, s>>>(d, nt, counts, base, offsets, (int32_t*)(ws + p.tiles),
                                             (int32_t*)(ws + p.ntiles));
  dispatch_scatter_kernel<<<nt, kDispatchThreads, 0, s>>>(d, idx, base, perm, rowmeta, topk_w);
  count_launches(3);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_fused(const Dims& d, const int32_t* idx, const int32_t* counts, const WsPlan& p, char* ws,
                                  int32_t* offsets, int32_t* perm, const float* topk_w, cudaStream_t s) {
  const cudaError_t e = launch_dependent(dispatch_fused_kernel, dim3(dispatch_tiles(d)), dim3(kDispatchThreads), 0, s,
                                         1, d, idx, counts, offsets, perm, (int32_t*)(ws + p.tiles),
                                         (int32_t*)(ws + p.ntiles), (int2*)(ws + p.rowmeta), topk_w);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_dispatch_gather(const Dims& d, const int32_t* idx, const int32_t* counts, const WsPlan& p, char* ws,
                                   int32_t* offsets, int32_t* perm, const float* topk_w, const void* X,
                                   cudaStream_t s) {
  // CTAs per tile: 8 (each CTA ranks its whole tile, so more CTAs cost more redundant ranking), up to 32
  // when there are so few tiles that 8 per tile would leave most SMs idle
  static int nsm = 0;
  if (nsm == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) !=
                                                   cudaSuccess)
      nsm = 148;
  }
  const int nt = dispatch_tiles(d);
  int split = 8;
  while (split < 32 && nt * split < nsm / 2) split *= 2;
  const cudaError_t e = launch_dependent(
      dispatch_gather_kernel<__nv_bfloat16>, dim3(nt * split), dim3(kDispatchThreads), 0, s, 1, d, idx, counts, offsets,
      perm, (int32_t*)(ws + p.tiles), (int32_t*)(ws + p.ntiles), (int2*)(ws + p.rowmeta), topk_w,
      (const __nv_bfloat16*)X, (__nv_bfloat16*)(ws + p.xsorted), split);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_gather_rows(const Dims& d, const void* X, const int32_t* perm, void* xsorted, cudaStream_t s) {
  const int rows = d.M * d.k;
  dim3 grid(ceil_div(rows, 8));
  cudaError_t e;
  if (d.dtype == SWIMBA_BF16)
    e = launch_dependent(gather_rows_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, 1, d, (const __nv_bfloat16*)X, perm,
                         (__nv_bfloat16*)xsorted);
  else
    e = launch_dependent(gather_rows_kernel<float>, grid, dim3(256), 0, s, 1, d, (const float*)X, perm,
                         (float*)xsorted);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace swimba
