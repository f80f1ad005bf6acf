// Grouped expert projection on the 5th-generation tensor cores, with the parameter-space mix fused into
// the epilogue (bf16 inputs, fp32 accumulation in TMEM, fp16 streams out).
//
// Paper: Swimba notes, key design 1 -- every active expert e projects X_t into its candidate streams
// (x^(e), B^(e), C^(e)) which are mixed with the router weights before the single recurrence:
//   Xs[m][j] = x^(j),   Bpi[m][j] = pi_mj B^(j),   Cpi[m][j] = pi_mj C^(j).
// The notes name a fused MoE operator for this input projection as the way to avoid HBM round trips of
// router outputs and parameter slices; here the per-expert output tile never leaves the SM unmixed.
//
// Design (one persistent CTA per SM, 14 warps):
//   warp 0      TMA producer: A = 128 gathered X rows x 64 K (16 KB), B = 256 weight rows x 64 K (32 KB)
//               per stage, 128-byte swizzle, kStages-deep ring of mbarriers
//   warp 1      TMEM owner and MMA issuer: 4 x tcgen05.mma M128 N256 K16 per stage into one of two
//               256-column fp32 accumulators (double buffered: 512 TMEM columns)
//   warps 2..13 epilogue: warp w reads TMEM lanes 32*(w%4).. and one column part of the tile (96, 96 or
//               64 columns), 32 columns at a time; scales B and C columns by pi, converts to fp16 and stores to the
//               destination (token, slot) row.  Each row's (pair, pi) comes from the dispatch's per-row
//               metadata in one load issued before the accumulator wait; the next tile's schedule entry
//               is prefetched while the current tile drains.
// Tiles: (row tile of one expert's sorted rows) x (256 output columns), handed out round-robin.
#include "tc_common.cuh"

namespace swimba {

namespace {
constexpr int BM = 128, BN = 256, BK = 64, kStages = 4;
constexpr int kEpiWarps = 12;                             // 3 per TMEM lane quarter
constexpr int kEpiParts = kEpiWarps / 4;                  // column parts of a tile
constexpr int kChunks = BN / 32;                          // 32-column chunks of a tile row
constexpr int kChunksPerPart = (kChunks + kEpiParts - 1) / kEpiParts;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kStageA = BM * BK * 2, kStageB = BN * BK * 2, kStageBytes = kStageA + kStageB;
constexpr uint32_t kTmemCols = 2 * BN;
constexpr uint32_t kIdesc = tc::idesc_f16(BM, BN, /*bf16=*/true);
constexpr int kStageRow = 80;                             // 64 B of fp16 + 16 B pad (conflict-free)
constexpr uint32_t kEpiStage = 32 * kStageRow;            // one warp's 32 rows x 32 columns
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 1024 + (size_t)kEpiWarps * kEpiStage;

struct TcArgs {
  Dims d;
  const int2* rowmeta;  // per sorted row: (pair index, router weight bits)
  const int32_t* tiles;
  const int32_t* ntiles;
  const int32_t* offsets;
  int mode;  // 0 mix, 1 mix with unscaled B, 2 raw fp32 Z, 3 plain bf16 product (the output projection),
             // 4 mix plus the raw fp32 B and C columns of Z (the layer gradients' forward recompute)
  int dense;  // 1: one operand group over rows 0 .. M-1 in order (no dispatch schedule, offsets or row metadata)
  __half* bpi;
  __half* xs;
  __half* cpi;
  float* Z;
  unsigned* st;
  __nv_bfloat16* out;  // mode 3: [M][We] bf16
};

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

// Write the 32 accumulator values of one row (columns c0 .. c0+31 of z = [x | B | C]) to their stream.
__device__ __forceinline__ void store_chunk(const TcArgs& a, int p, float pi, int c0, const uint32_t (&r)[32],
                                           bool& range_bad) {
  const Dims& d = a.d;
  if (a.mode == 2) {
    float* dst = a.Z + (size_t)p * d.We + c0;
    if (c0 + 32 <= d.We) {
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4*>(dst + i) = make_float4(u2f(r[i]), u2f(r[i + 1]), u2f(r[i + 2]), u2f(r[i + 3]));
    } else {
      for (int i = 0; i < 32 && c0 + i < d.We; ++i) dst[i] = u2f(r[i]);
    }
    return;
  }
  const int HP = d.HP, GN = d.GN;
  auto stream_of = [&](int c) { return c < HP ? 0 : (c < HP + GN ? 1 : 2); };
  const int s0 = stream_of(c0);
  if (c0 + 32 <= d.We && stream_of(c0 + 31) == s0) {
    __half* dst;
    float sc;
    if (s0 == 0) { dst = a.xs + (size_t)p * HP + c0; sc = 1.f; }
    else if (s0 == 1) { dst = a.bpi + (size_t)p * GN + (c0 - HP); sc = a.mode == 1 ? 1.f : pi; }
    else { dst = a.cpi + (size_t)p * GN + (c0 - HP - GN); sc = pi; }
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
      uint4 v;
      uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float f0 = sc * u2f(r[i + 2 * q]), f1 = sc * u2f(r[i + 2 * q + 1]);
        range_bad |= !(fabsf(f0) <= kF16Max) || !(fabsf(f1) <= kF16Max);
        __half2 h = __floats2half2_rn(f0, f1);
        w[q] = *reinterpret_cast<uint32_t*>(&h);
      }
      *reinterpret_cast<uint4*>(dst + i) = v;
    }
    return;
  }
  for (int i = 0; i < 32; ++i) {
    const int c = c0 + i;
    if (c >= d.We) break;
    const int s = stream_of(c);
    const float v = u2f(r[i]);
    float o;
    __half* dst;
    if (s == 0) { o = v; dst = a.xs + (size_t)p * HP + c; }
    else if (s == 1) { o = a.mode == 1 ? v : pi * v; dst = a.bpi + (size_t)p * GN + (c - HP); }
    else { o = pi * v; dst = a.cpi + (size_t)p * GN + (c - HP - GN); }
    range_bad |= !(fabsf(o) <= kF16Max);
    *dst = __float2half_rn(o);
  }
}

// Mode 4: the raw B and C columns (W_e columns from H*P on) of one row's 32-column group, fp32 into row p of
// Z [M*k][W_e]; the x columns are not stored (the mix's gradient does not read them).
__device__ __forceinline__ void store_raw_bc(const TcArgs& a, int p, int c0, const uint32_t (&r)[32]) {
  const Dims& d = a.d;
  float* dst = a.Z + (size_t)p * d.We + c0;
  if (c0 >= d.HP && c0 + 32 <= d.We) {
#pragma unroll
    for (int i = 0; i < 32; i += 4)
      *reinterpret_cast<float4*>(dst + i) = make_float4(u2f(r[i]), u2f(r[i + 1]), u2f(r[i + 2]), u2f(r[i + 3]));
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)  // constant indices keep r in registers
      if (c0 + i >= d.HP && c0 + i < d.We) dst[i] = u2f(r[i]);
  }
}

// Destination of the 32-column group starting at column c0 of z when it lies in one stream (else null),
// and the scale its values take.
__device__ __forceinline__ __half* group_dst(const TcArgs& a, int p, float pi, int c0, float& sc) {
  const Dims& d = a.d;
  const int HP = d.HP, GN = d.GN;
  if (c0 + 32 > d.We) return nullptr;
  if (c0 + 32 <= HP) { sc = 1.f; return a.xs + (size_t)p * HP + c0; }
  if (c0 >= HP && c0 + 32 <= HP + GN) { sc = a.mode == 1 ? 1.f : pi; return a.bpi + (size_t)p * GN + (c0 - HP); }
  if (c0 >= HP + GN) { sc = pi; return a.cpi + (size_t)p * GN + (c0 - HP - GN); }
  return nullptr;
}

// One warp stores 32 columns of its 32 rows: each thread converts its row's values to fp16 into the warp's
// staging rows, then every store instruction writes 8 whole 64-byte row segments.
__device__ __forceinline__ void store_group32(const TcArgs& a, uint8_t* stage, int lane, bool valid, int p, float pi,
                                              int c0, const uint32_t (&r)[32], bool& range_bad) {
  float sc = 0.f;
  __half* dst = valid ? group_dst(a, p, pi, c0, sc) : nullptr;
  uint8_t* my = stage + lane * kStageRow;
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    uint4 v;
    uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float f0 = sc * u2f(r[i + 2 * q]), f1 = sc * u2f(r[i + 2 * q + 1]);
      range_bad |= dst && (!(fabsf(f0) <= kF16Max) || !(fabsf(f1) <= kF16Max));
      __half2 h = __floats2half2_rn(f0, f1);
      w[q] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(my + 2 * i) = v;
  }
  __syncwarp();
  const unsigned long long dptr = reinterpret_cast<unsigned long long>(dst);
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int row = 8 * it + (lane >> 2), chunk = lane & 3;
    const unsigned long long rd = __shfl_sync(0xffffffffu, dptr, row);
    if (rd) *reinterpret_cast<uint4*>(rd + 16 * chunk) = *reinterpret_cast<const uint4*>(stage + row * kStageRow + 16 * chunk);
  }
  __syncwarp();
}

// Mode 3: one warp stores 32 columns of its 32 rows of the plain product as bf16 (row-major [M][We]), staged
// through shared memory so that every store instruction writes 8 whole 64-byte row segments; a ragged last
// column group is stored per thread.
__device__ __forceinline__ void store_dense32(const TcArgs& a, uint8_t* stage, int lane, bool valid, int row, int c0,
                                              const uint32_t (&r)[32]) {
  const int N = a.d.We;
  if (c0 + 32 > N) {
#pragma unroll
    for (int i = 0; i < 32; ++i)  // constant indices keep r in registers
      if (valid && c0 + i < N) a.out[(size_t)row * N + c0 + i] = __float2bfloat16_rn(u2f(r[i]));
    return;
  }
  uint8_t* my = stage + lane * kStageRow;
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    uint4 v;
    uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __nv_bfloat162 h = __floats2bfloat162_rn(u2f(r[i + 2 * q]), u2f(r[i + 2 * q + 1]));
      w[q] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(my + 2 * i) = v;
  }
  __syncwarp();
  const unsigned long long dptr = valid ? reinterpret_cast<unsigned long long>(a.out + (size_t)row * N + c0) : 0ull;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int rr = 8 * it + (lane >> 2), chunk = lane & 3;
    const unsigned long long rd = __shfl_sync(0xffffffffu, dptr, rr);
    if (rd) *reinterpret_cast<uint4*>(rd + 16 * chunk) = *reinterpret_cast<const uint4*>(stage + rr * kStageRow + 16 * chunk);
  }
  __syncwarp();
}

// One epilogue warp drains its 32 accumulator rows x nch 32-column chunks (starting at output column col0)
// of a tile: the TMEM load of the next chunk is in flight while the current one is converted and stored.
// kRaw: mode 4, whose raw B/C stores are compiled only into the kernels that run it.
template <bool kRaw>
__device__ __forceinline__ void drain_tile(const TcArgs& a, uint32_t taddr, int col0, int nch, bool valid, int2 meta,
                                           uint8_t* stage, int lane, bool& range_bad) {
  const Dims& d = a.d;
  const float pi = __int_as_float(meta.y);
  uint32_t ra[32], rb[32];
  tc::tmem_ld_32x32b_x32(taddr, ra);
#pragma unroll
  for (int c = 0; c < kChunksPerPart; ++c) {
    if (c >= nch) break;
    uint32_t(&cur)[32] = (c & 1) ? rb : ra;
    uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
    tc::tmem_ld_wait(cur);
    if (c + 1 < nch) tc::tmem_ld_32x32b_x32(taddr + 32 * (c + 1), nxt);
    const int c0 = col0 + 32 * c;
    if (a.mode == 3) {
      store_dense32(a, stage, lane, valid, meta.x, c0, cur);
      continue;
    }
    if (kRaw && valid && c0 + 32 > d.HP && c0 < d.We) store_raw_bc(a, meta.x, c0, cur);
    float sc_probe;
    // fast path: the warp's 32-column group lies in one fp16 stream for every valid row
    const bool fast = a.mode != 2 && c0 + 32 <= d.We &&
                      __all_sync(0xffffffffu, !valid || group_dst(a, meta.x, pi, c0, sc_probe) != nullptr);
    if (fast) store_group32(a, stage, lane, valid, meta.x, pi, c0, cur, range_bad);
    else if (valid && c0 < d.We) store_chunk(a, meta.x, pi, c0, cur, range_bad);
  }
}

template <bool kRaw>
__global__ void __launch_bounds__(kThreads, 1)
proj_tc_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b, TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* full = bars;                 // [kStages]  TMA -> MMA
  uint64_t* empty = bars + kStages;      // [kStages]  MMA -> TMA
  uint64_t* acc_full = bars + 2 * kStages;       // [2]  MMA -> epilogue
  uint64_t* acc_empty = bars + 2 * kStages + 2;  // [2]  epilogue -> MMA
  uint64_t* drain = bars + 2 * kStages + 4;      // MMA completion before teardown
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* off_s = reinterpret_cast<int*>(tmem_slot + 2);  // [E + 1] expert offsets

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Dims& d = a.d;
  const int nct = ceil_div(d.We, BN);
  const int nkb = ceil_div(d.D, BK);  // a dense product's ragged K tail is zero-filled by TMA

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { tc::mbar_init(&full[s], 1); tc::mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&acc_full[b], 1); tc::mbar_init(&acc_empty[b], 32 * kEpiWarps); }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tmap_a);
    tc::tma_prefetch_desc(&tmap_b);
  }
  griddep_launch_dependents();
  if (warp == 1) { tc::tmem_alloc(tmem_slot, kTmemCols); tc::tmem_relinquish(); }
  griddep_wait();  // the dispatch's offsets and schedule, the gathered rows
  if (a.dense) {
    if (threadIdx.x == 0) { off_s[0] = 0; off_s[1] = d.M; }
  } else {
    for (int e = threadIdx.x; e <= d.E; e += blockDim.x) off_s[e] = a.offsets[e];
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int total = (a.dense ? ceil_div(d.M, BM) : *a.ntiles) * nct;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const int rt = t / nct, ct = t % nct;
      const int e = a.dense ? 0 : a.tiles[2 * rt], row0 = a.dense ? rt * BM : a.tiles[2 * rt + 1];
      const int wrow = e * d.We + ct * BN;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!tc::mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        uint8_t* sa = stage_base + stage * kStageBytes;
        tc::mbar_arrive_expect_tx(&full[stage], kStageBytes);
        tc::tma_load_2d(sa, &tmap_a, &full[stage], kb * BK, row0);
        tc::tma_load_2d(sa + kStageA, &tmap_b, &full[stage], kb * BK, wrow);
        ++issued;
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok) { *abort_flag = 1; atomicOr(a.st, ST_TIMEOUT); }
    // make sure every copy this CTA issued has landed before the CTA can exit
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
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      if (!tc::mbar_wait(&acc_empty[buf], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
      tc::fence_after_sync();
      const uint32_t dt = tmem + (uint32_t)(buf * BN);
      for (int kb = 0; kb < nkb; ++kb) {
        if (!tc::mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t sa = tc::smem_u32(stage_base + stage * kStageBytes);
        const uint64_t da = tc::sdesc_kmajor_sw128(sa), db = tc::sdesc_kmajor_sw128(sa + kStageA);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)  // K16 step: +32 bytes = +2 in the descriptor's address field
          tc::mma_f16(dt, da + 2 * kk, db + 2 * kk, kIdesc, (kb | kk) != 0);
        tc::mma_commit(&empty[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      tc::mma_commit(&acc_full[buf]);
      if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
    }
    if (!ok) { *abort_flag = 1; atomicOr(a.st, ST_TIMEOUT); }
    tc::mma_commit(drain);
    volatile int never = 0;
    tc::mbar_wait(drain, 0, &never);
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int part = (warp - 2) >> 2;    // which column part of the tile (chunks part*3 .. , 3 / 3 / 2)
    const int ch0 = part * kChunksPerPart, nch = min(kChunksPerPart, kChunks - ch0);
    const int row_local = 32 * q + lane;
    uint8_t* epi_stage = smem + kStages * kStageBytes + 1024 + (warp - 2) * kEpiStage;
    int buf = 0;
    uint32_t acc_phase = 0;
    bool range_bad = false;
    int t = blockIdx.x;
    auto tile_info = [&](int tt) {
      return a.dense ? make_int2(0, (tt / nct) * BM) : *reinterpret_cast<const int2*>(a.tiles + 2 * (tt / nct));
    };
    int2 tinfo = t < total ? tile_info(t) : make_int2(0, 0);
    for (; t < total; t += gridDim.x) {
      const int ct = t % nct;
      const int e = tinfo.x, row0 = tinfo.y;
      const bool valid = row0 + row_local < off_s[e + 1];
      const int2 meta = !valid ? make_int2(0, 0) : (a.dense ? make_int2(row0 + row_local, 0) : a.rowmeta[row0 + row_local]);
      const int tn = t + gridDim.x;
      if (tn < total) tinfo = tile_info(tn);
      if (!tc::mbar_wait(&acc_full[buf], acc_phase, abort_flag)) {
        *abort_flag = 1;
        atomicOr(a.st, ST_TIMEOUT);
        break;
      }
      tc::fence_after_sync();
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN + 32 * ch0);
      drain_tile<kRaw>(a, taddr, ct * BN + 32 * ch0, nch, valid, meta, epi_stage, lane, range_bad);
      tc::fence_before_sync();
      tc::mbar_arrive(&acc_empty[buf]);
      if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
    }
    if (range_bad) atomicOr(a.st, ST_RANGE);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------
// CTA-pair variant: a cluster of 2 CTAs computes one 256-row x 256-column tile with tcgen05.mma
// cta_group::2 (M256 N256 K16).  Each CTA loads 128 gathered X rows and 128 of the 256 weight rows per
// 64-wide K slice (32 KB per stage instead of 48 KB for half the FLOPs of a 128 x 256 tile per CTA), so a
// stage's copies keep pace with the tensor pipe.  The even CTA's producer arms its full barrier for both
// CTAs' bytes; the odd CTA's copies complete on that barrier.  The even CTA's warp 1 issues the MMAs and
// its commits arrive on both CTAs' barriers (stage free, accumulator ready); both CTAs drain their own
// 128 accumulator rows with the same epilogue as above and tell the even CTA's MMA warp when a buffer is
// free.  Tiles: 256 consecutive sorted rows of one expert (rows past the expert's end are computed and
// dropped) x 256 output columns; the pair-tile schedule is derived from the expert offsets in the kernel.
constexpr int kPairStages = 6;
constexpr uint32_t kPairStageA = 128 * BK * 2, kPairStageB = 128 * BK * 2;
constexpr uint32_t kPairStageBytes = kPairStageA + kPairStageB;
constexpr uint32_t kPairIdesc = tc::idesc_f16(256, BN, /*bf16=*/true);
constexpr size_t kPairSmemBytes = 1024 + (size_t)kPairStages * kPairStageBytes + 1024 + (size_t)kEpiWarps * kEpiStage;
constexpr int kPairRows = 256;

// Pair tile rt -> (expert, first sorted row), from pt_s[e] = number of 256-row tiles of experts < e.
__device__ __forceinline__ int2 pair_tile(const int* off_s, const int* pt_s, int E, int rt) {
  int e = 0;
  while (e + 1 < E && pt_s[e + 1] <= rt) ++e;
  return make_int2(e, off_s[e] + (rt - pt_s[e]) * kPairRows);
}

template <bool kRaw>
__global__ void __launch_bounds__(kThreads, 1)
proj_tc_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b, TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPairStages * kPairStageBytes);
  uint64_t* full = bars;                               // [kPairStages] copies of both CTAs -> MMA (even CTA)
  uint64_t* empty = bars + kPairStages;                // [kPairStages] MMA -> this CTA's producer
  uint64_t* acc_full = bars + 2 * kPairStages;         // [2] MMA -> this CTA's epilogue
  uint64_t* acc_empty = bars + 2 * kPairStages + 2;    // [2] both epilogues -> MMA (even CTA)
  uint64_t* drain = bars + 2 * kPairStages + 4;        // all MMAs complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kPairStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* off_s = reinterpret_cast<int*>(tmem_slot + 2);  // [E + 1] expert offsets
  int* pt_s = off_s + 65;                               // [E + 1] pair-tile prefix

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_ctarank();
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  const Dims& d = a.d;
  const int nct = ceil_div(d.We, BN);
  const int nkb = ceil_div(d.D, BK);  // a dense product's ragged K tail is zero-filled by TMA

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) { tc::mbar_init(&full[s], 1); tc::mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&acc_full[b], 1); tc::mbar_init(&acc_empty[b], 2 * kEpiWarps); }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tmap_a);
    tc::tma_prefetch_desc(&tmap_b);
  }
  griddep_launch_dependents();
  if (warp == 1) { tc::tmem_alloc_pair(tmem_slot, kTmemCols); tc::tmem_relinquish_pair(); }
  griddep_wait();  // the dispatch's offsets, the gathered rows
  if (a.dense) {
    if (threadIdx.x == 0) { off_s[0] = 0; off_s[1] = d.M; }
  } else {
    for (int e = threadIdx.x; e <= d.E; e += blockDim.x) off_s[e] = a.offsets[e];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < d.E; ++e) { pt_s[e] = acc; acc += ceil_div(off_s[e + 1] - off_s[e], kPairRows); }
    pt_s[d.E] = acc;
  }
  tc::fence_before_sync();
  tc::cluster_sync();  // both CTAs' barriers are initialised before any copy or commit can reach them
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int total = pt_s[d.E] * nct;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    bool ok = true;
    const uint32_t full0 = tc::map_shared(tc::smem_u32(full), 0u);  // the even CTA's full barriers
    for (int t = cid; t < total && ok; t += ncl) {
      const int rt = t / nct, ct = t % nct;
      const int2 tl = pair_tile(off_s, pt_s, d.E, rt);
      const int arow = tl.y + 128 * (int)rank;
      const int wrow = tl.x * d.We + ct * BN + 128 * (int)rank;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!tc::mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        uint8_t* sa = stage_base + stage * kPairStageBytes;
        if (rank == 0) tc::mbar_arrive_expect_tx(&full[stage], 2 * kPairStageBytes);
        const uint32_t fb = full0 + 8u * (uint32_t)stage;
        tc::tma_load_2d_pair(sa, &tmap_a, fb, kb * BK, arow);
        tc::tma_load_2d_pair(sa + kPairStageA, &tmap_b, fb, kb * BK, wrow);
        ++issued;
        if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok) { *abort_flag = 1; atomicOr(a.st, ST_TIMEOUT); }
    // every copy this CTA issued has been consumed by an MMA (its stage was released) or is waited for here
    for (long long i = 0; i < kPairStages && i < issued; ++i) {
      if (--stage < 0) { stage = kPairStages - 1; phase ^= 1u; }
      volatile int never = 0;
      tc::mbar_wait(&empty[stage], phase, &never);
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ---------------------------------------------------------------- MMA issuer (even CTA)
    int stage = 0;
    uint32_t phase = 0;
    int buf = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int t = cid; t < total && ok; t += ncl) {
      if (!tc::mbar_wait(&acc_empty[buf], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
      tc::fence_after_sync();
      const uint32_t dt = tmem + (uint32_t)(buf * BN);
      for (int kb = 0; kb < nkb; ++kb) {
        if (!tc::mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t sa = tc::smem_u32(stage_base + stage * kPairStageBytes);
        const uint64_t da = tc::sdesc_kmajor_sw128(sa), db = tc::sdesc_kmajor_sw128(sa + kPairStageA);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)  // K16 step: +32 bytes = +2 in the descriptor's address field
          tc::mma_f16_pair(dt, da + 2 * kk, db + 2 * kk, kPairIdesc, (kb | kk) != 0);
        tc::mma_commit_pair(&empty[stage], 0x3);
        if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      tc::mma_commit_pair(&acc_full[buf], 0x3);
      if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
    }
    if (!ok) { *abort_flag = 1; atomicOr(a.st, ST_TIMEOUT); }
    tc::mma_commit_pair(drain, 0x3);
    volatile int never = 0;
    tc::mbar_wait(drain, 0, &never);
  } else if (warp == 1 && lane == 0) {
    // odd CTA: its TMEM and shared memory are in use until the even CTA's last MMA has completed
    volatile int never = 0;
    tc::mbar_wait(drain, 0, &never);
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;
    const int ch0 = part * kChunksPerPart, nch = min(kChunksPerPart, kChunks - ch0);
    const int row_local = 128 * (int)rank + 32 * q + lane;  // row inside the 256-row pair tile
    uint8_t* epi_stage = smem + kPairStages * kPairStageBytes + 1024 + (warp - 2) * kEpiStage;
    const uint32_t acc_empty0 = tc::map_shared(tc::smem_u32(acc_empty), 0u);
    int buf = 0;
    uint32_t acc_phase = 0;
    bool range_bad = false;
    for (int t = cid; t < total; t += ncl) {
      const int rt = t / nct, ct = t % nct;
      const int2 tl = pair_tile(off_s, pt_s, d.E, rt);
      const bool valid = tl.y + row_local < off_s[tl.x + 1];
      const int2 meta = !valid ? make_int2(0, 0) : (a.dense ? make_int2(tl.y + row_local, 0) : a.rowmeta[tl.y + row_local]);
      if (!tc::mbar_wait(&acc_full[buf], acc_phase, abort_flag)) {
        *abort_flag = 1;
        atomicOr(a.st, ST_TIMEOUT);
        break;
      }
      tc::fence_after_sync();
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * BN + 32 * ch0);
      drain_tile<kRaw>(a, taddr, ct * BN + 32 * ch0, nch, valid, meta, epi_stage, lane, range_bad);
      // the accumulator's TMEM reads are complete (tcgen05.wait::ld) and ordered by the tcgen05 fence; the
      // tile's global stores need not be visible to the even CTA, so the arrival is relaxed
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive_cluster_relaxed(acc_empty0 + 8u * (uint32_t)buf);
      if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
    }
    if (range_bad) atomicOr(a.st, ST_RANGE);
  }
  tc::fence_before_sync();
  tc::cluster_sync();  // no CTA leaves while the other may still signal its barriers or read its operands
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace

// Host side --------------------------------------------------------------------------------------
// The CTA-pair kernel, persistent: as many pairs as can be resident at once, at most one per pair tile.
template <bool kRaw>
static cudaError_t launch_pair(const CUtensorMap& ta, const CUtensorMap& tb2, const TcArgs& a, int max_pairs, int sms,
                               cudaStream_t s) {
  cudaError_t e = set_max_dynamic_smem((const void*)proj_tc_pair_kernel<kRaw>, kPairSmemBytes);
  if (e != cudaSuccess) return e;
  static int resident = 0;
  if (resident == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kPairSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)sms);
    int n = 0;
    resident = cudaOccupancyMaxActiveClusters(&n, proj_tc_pair_kernel<kRaw>, &cfg) == cudaSuccess && n > 0 ? n : sms / 2;
  }
  const int pairs = resident < max_pairs ? resident : max_pairs;
  return launch_dependent(proj_tc_pair_kernel<kRaw>, dim3((unsigned)(2 * pairs)), dim3(kThreads), kPairSmemBytes, s, 2, ta,
                          tb2, a);
}

template <bool kRaw>
static cudaError_t launch_proj_tc_t(const Dims& d, const void* xsorted, const void* w_exp, const int2* rowmeta,
                                   const int32_t* tiles, const int32_t* ntiles, const int32_t* offsets, int mode,
                                   void* bpi, void* xs, void* cpi, float* Z, unsigned* st, cudaStream_t s) {
  CUtensorMap ta, tb;
  if (!encode_tmap_2d(&ta, xsorted, SWIMBA_BF16, (uint64_t)d.D, (uint64_t)d.M * d.k, (uint64_t)d.D * 2, BK, BM))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d(&tb, w_exp, SWIMBA_BF16, (uint64_t)d.D, (uint64_t)d.E * d.We, (uint64_t)d.D * 2, BK, BN))
    return cudaErrorInvalidValue;
  TcArgs a{d, rowmeta, tiles, ntiles, offsets, mode, 0, (__half*)bpi, (__half*)xs, (__half*)cpi, Z, st, nullptr};
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e;
  // CTA pairs when experts average at least 1536 rows: each expert's last pair tile is partly past its
  // rows, and below that the 256-row tiles waste more tensor time than the pairs' lower operand traffic
  // (a third less per FLOP from L2) saves
  if ((long long)d.M * d.k >= 1536LL * d.E) {
    // CTA pairs: A boxes of 128 rows (the pair's two halves), B boxes of 128 weight rows
    CUtensorMap tb2;
    if (!encode_tmap_2d(&tb2, w_exp, SWIMBA_BF16, (uint64_t)d.D, (uint64_t)d.E * d.We, (uint64_t)d.D * 2, BK, 128))
      return cudaErrorInvalidValue;
    e = launch_pair<kRaw>(ta, tb2, a, (ceil_div(d.M * d.k, kPairRows) + d.E) * ceil_div(d.We, BN), sms, s);
    if (e == cudaSuccess) {
      count_launches(1);
      return cudaGetLastError();
    }
    (void)cudaGetLastError();  // pairs could not be launched: the one-CTA kernel below does the work
  }
  e = set_max_dynamic_smem((const void*)proj_tc_kernel<kRaw>, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int max_tiles = max_row_tiles(d) * ceil_div(d.We, BN);
  const int grid = max_tiles < sms ? max_tiles : sms;
  e = launch_dependent(proj_tc_kernel<kRaw>, dim3(grid), dim3(kThreads), kSmemBytes, s, 1, ta, tb, a);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_proj_tc(const Dims& d, const void* xsorted, const void* w_exp, const int2* rowmeta,
                           const int32_t* tiles, const int32_t* ntiles, const int32_t* offsets, int mode, void* bpi,
                           void* xs, void* cpi, float* Z, unsigned* st, cudaStream_t s) {
  return mode == 4 ? launch_proj_tc_t<true>(d, xsorted, w_exp, rowmeta, tiles, ntiles, offsets, mode, bpi, xs, cpi, Z,
                                            st, s)
                   : launch_proj_tc_t<false>(d, xsorted, w_exp, rowmeta, tiles, ntiles, offsets, mode, bpi, xs, cpi,
                                             Z, st, s);
}

// The output projection out = y W_out^T as one dense product on the one-CTA kernel: A = y [M][K] (K = H*P),
// B = W_out [N][K] (N = d_model), out [M][N] bf16.  K must be a multiple of 64, N of 8.
cudaError_t launch_out_proj_tc(int M, int K, int N, const void* y, const void* w_out, void* out, unsigned* st,
                               cudaStream_t s) {
  CUtensorMap ta, tb;
  if (!encode_tmap_2d(&ta, y, SWIMBA_BF16, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, BK, BM))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d(&tb, w_out, SWIMBA_BF16, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, BK, BN))
    return cudaErrorInvalidValue;
  Dims d{};
  d.M = M; d.D = K; d.We = N; d.E = 1; d.k = 1; d.dtype = SWIMBA_BF16;
  TcArgs a{d, nullptr, nullptr, nullptr, nullptr, 3, 1, nullptr, nullptr, nullptr, nullptr, st,
           (__nv_bfloat16*)out};
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e;
  // CTA pairs (256-row tiles, half the operand bytes per FLOP) once there are rows for a few pair tiles
  if (M >= 4 * kPairRows) {
    CUtensorMap tb2;
    if (!encode_tmap_2d(&tb2, w_out, SWIMBA_BF16, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, BK, 128))
      return cudaErrorInvalidValue;
    e = launch_pair<false>(ta, tb2, a, ceil_div(M, kPairRows) * ceil_div(N, BN), sms, s);
    if (e == cudaSuccess) {
      count_launches(1);
      return cudaGetLastError();
    }
    (void)cudaGetLastError();  // pairs could not be launched: the one-CTA kernel below does the work
  }
  e = set_max_dynamic_smem((const void*)proj_tc_kernel<false>, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int tiles = ceil_div(M, BM) * ceil_div(N, BN);
  e = launch_dependent(proj_tc_kernel<false>, dim3(tiles < sms ? tiles : sms), dim3(kThreads), kSmemBytes, s, 1, ta, tb, a);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace swimba
