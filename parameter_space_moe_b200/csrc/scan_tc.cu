// Chunked solve of the single shared-transition recurrence on the tensor cores (fp16 streams, fp32
// accumulation and state), with the inter-chunk state pass chained between CTAs.
//
// Paper: Swimba notes, key design 1 (h_t = a_t h_{t-1} + U~_t, y_t = C~_t^T h_t, U~_t = sum_j Bpi_tj Xs_tj^T)
// and the overall framework's chunked SSD solve.  One CTA owns SUB = 128 consecutive tokens of one
// (sequence, head); with cs_t the running sum of dt*A from the sub-chunk start:
//   S_j      = C~ Bpi_j^T                        (tensor core, 128 x 128 per key slot j, in TMEM)
//   Pm_j     = mask_{s<=t}(S_j * exp(cs_t - cs_s))   (registers -> fp16 pairs back into TMEM over S_j)
//   Y       += Pm_j Xs_j                          (tensor core, Pm_j read from TMEM)
//   Sc      += Bpi_j^T (exp(cs_end - cs_s) Xs_j)  (tensor core: the sub-chunk's own end state)
//   H_out    = exp(cs_end) H_in + Sc              (fp32; H_in from the previous sub-chunk's CTA)
//   y        = Y + exp(cs_t) C~ H_in              (tensor core, H_in split into fp16 hi + lo parts)
// The hand-off: CTAs take tickets in launch order, ticket -> (sub-chunk = ticket / (B*H), head row =
// ticket % (B*H)), so the CTA holding the previous sub-chunk of the same head always took its ticket
// first and is running or done.  It publishes H_out with a release flag; the successor polls with a
// bounded wait (on expiry it records ST_TIMEOUT, uses a zero state and still publishes its own flag).
// Keys are the (token, slot) pairs; the k slots are processed one after another, the next slot's keys
// and values loaded by TMA as soon as the current slot's products no longer read them.
#include "tc_common.cuh"

namespace swimba {

namespace {
constexpr int SUB = 128;
constexpr int kThreads = 256;
constexpr uint32_t kBlk = SUB * 128;  // one 64-wide column block of 128 swizzled 128-byte rows
constexpr uint32_t kFlagPolls = 1u << 22;

struct TcScanArgs {
  Dims d;
  const float* dt;
  const float* A;
  const float* init;
  const __half* cpi;
  __nv_bfloat16* y;
  float* final_state;
  float* chunk_states;
  float* exch;
  unsigned* flags;
  unsigned* ticket;
  unsigned* st;
  float* ysum;
  int nsub;
  int key_slot0, key_slots, read_slot0, read_slots;
  int accumulate_y, first_pass, last_pass;
};

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(tc::smem_u32(dst)),
      "l"((uint64_t)map), "r"(tc::smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_relaxed(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Shared-memory plan of one CTA (byte offsets from a 1024-aligned base).  With P = 64 it is 96 KB,
// so two CTAs share an SM and one CTA's loads overlap the other's tensor-core work.
template <int P>
struct ScanSmem {
  static constexpr int N = 128, NB = N / 64, PB = P / 64;
  static constexpr uint32_t CT = 0;               // C~ rows, K-major, NB blocks
  static constexpr uint32_t BP = CT + NB * kBlk;  // Bpi_j (NB blocks); H_in hi/lo parts after the slot loop
  static constexpr uint32_t XS = BP + NB * kBlk;  // Xs_j of even slots / decay-scaled Xs_j of odd slots
  static constexpr uint32_t PM = XS + PB * kBlk;  // the other way round
  static constexpr uint32_t BAR = PM + PB * kBlk; // fullB, fullX, done, hbar, fullC
  static constexpr uint32_t CS = BAR + 64;        // cs[SUB], fs[SUB], wsum[4], misc[2]
  static constexpr uint32_t END = CS + 2 * SUB * 4 + 64;
  static constexpr size_t bytes() { return 1024 + END; }
};

// Thread layout: 8 warps; thread (row = tid % 128, half = tid / 128).  Warps w and w + 4 read the same
// TMEM lane quarter (w % 4) and split the columns of each row between them.
template <int P>
__global__ void __launch_bounds__(kThreads, P == 64 ? 2 : 1)
scan_tc_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_x,
               const __grid_constant__ CUtensorMap tm_c, TcScanArgs a) {
  using Lay = ScanSmem<P>;
  constexpr int N = 128, NB = Lay::NB, PB = Lay::PB, PH = P / 2;
  constexpr uint32_t TMEM_COLS = P == 64 ? 256 : 512;
  constexpr uint32_t COL_S = 0, COL_Y = 128, COL_SC = 128 + P;
  constexpr uint32_t ID_S = tc::idesc_f16(128, 128, false);
  constexpr uint32_t ID_SC = tc::idesc_f16(128, P, false, true, true);
  constexpr uint32_t ID_Y = tc::idesc_f16(128, P, false, false, true);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* CT = sm + Lay::CT;
  uint8_t* BP = sm + Lay::BP;
  uint8_t* XS = sm + Lay::XS;
  uint8_t* PM = sm + Lay::PM;
  uint64_t* fullB = reinterpret_cast<uint64_t*>(sm + Lay::BAR);
  uint64_t* fullX = fullB + 1;
  uint64_t* done = fullB + 2;
  uint64_t* hbar = fullB + 3;  // bulk copy of H_in into the Bpi region
  uint64_t* fullC = fullB + 4;  // first read slot of C~ into CT
  float* cs_s = reinterpret_cast<float*>(sm + Lay::CS);
  float* fs_s = cs_s + SUB;
  float* wsum = fs_s + SUB;
  uint32_t* misc = reinterpret_cast<uint32_t*>(wsum + 4);

  const Dims& d = a.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = tid & (SUB - 1), half = tid >> 7;
  if (tid == 0) {
    tc::mbar_init(fullB, 1);
    tc::mbar_init(fullX, 1);
    tc::mbar_init(done, 1);
    tc::mbar_init(hbar, 1);
    tc::mbar_init(fullC, 1);
    tc::fence_barrier_init();
    // the ticket counter and flags are cleared by earlier work in the stream: the ticket is taken once the
    // grid launched before this one has completed, so every earlier write is visible
    griddep_wait();
    misc[1] = atomicAdd(a.ticket, 1u);
  }
  if (warp == 0) { tc::tmem_alloc(&misc[0], TMEM_COLS); tc::tmem_relinquish(); }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = misc[0];
  const int BH = d.Bsz * d.H;
  const int ticket = (int)misc[1];
  if (ticket >= BH * a.nsub) {  // no sub-chunk left for this CTA (the counter started past zero)
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
      tc::fence_after_sync();
      tc::tmem_dealloc(misc[0], TMEM_COLS);
    }
    return;
  }
  const int csub = ticket / BH, bh = ticket % BH, b = bh / d.H, h = bh % d.H, g = h / d.hpg;
  const int t0 = csub * SUB, L = min(SUB, d.T - t0);
  const int row0 = b * d.T + t0;
  const int nk = a.key_slots;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  volatile int never = 0;
  int issuedB = 0, issuedX = 0;

  griddep_wait();  // the streams of the expert projection, dt of the router
  auto issue_b = [&](int i) {
    tc::mbar_arrive_expect_tx(fullB, NB * kBlk);
    for (int nb = 0; nb < NB; ++nb) tma_load_3d(BP + nb * kBlk, &tm_b, fullB, g * N + 64 * nb, a.key_slot0 + i, row0);
    ++issuedB;
  };
  auto issue_x = [&](int i) {
    tc::mbar_arrive_expect_tx(fullX, PB * kBlk);
    uint8_t* dst = (i & 1) ? PM : XS;
    for (int pb = 0; pb < PB; ++pb) tma_load_3d(dst + pb * kBlk, &tm_x, fullX, h * P + 64 * pb, a.key_slot0 + i, row0);
    ++issuedX;
  };
  if (tid == 0) {
    issue_b(0);
    issue_x(0);
    tc::mbar_arrive_expect_tx(fullC, NB * kBlk);
    for (int nb = 0; nb < NB; ++nb) tma_load_3d(CT + nb * kBlk, &tm_c, fullC, g * N + 64 * nb, a.read_slot0, row0);
  }
  // H_in of this sub-chunk is the previous sub-chunk's H_out.  With P = 64 it fits the Bpi region once the
  // last slot's key products are done, so thread 0 fetches it with one bulk copy as soon as the
  // predecessor's flag is up, while the other threads still work on the last slot.
  constexpr bool kEarlyFetch = P == 64;
  const size_t NPs = (size_t)N * P;
  const float* hprev = csub > 0 ? a.exch + ((size_t)bh * a.nsub + csub - 1) * NPs : nullptr;
  const unsigned* pflag = csub > 0 ? a.flags + (size_t)bh * a.nsub + csub - 1 : nullptr;
  bool h_issued = false;
  unsigned fpeek = 0u;  // thread 0: a relaxed read of the predecessor's flag, looked at one phase later
  auto fetch_hin = [&]() {
    tc::fence_proxy_async_global();
    tc::mbar_arrive_expect_tx(hbar, (uint32_t)(NPs * 4));
    tc::bulk_load(BP, hprev, (uint32_t)(NPs * 4), hbar);
    h_issued = true;
  };
  // during the last slot (thread 0 only): read the flag without waiting for the value, and one phase later
  // fetch H_in if it was up (the relaxed read that saw the release store plus fence.acq_rel is the acquire)
  auto peek_hin = [&]() {
    if (!kEarlyFetch || h_issued || csub == 0) return;
    if (fpeek) {
      fence_acq_rel_gpu();
      fetch_hin();
    } else {
      fpeek = ld_relaxed(pflag);
    }
  };
  auto wait_fetch_hin = [&]() {  // thread 0 only, at the hand-off
    if (!kEarlyFetch || h_issued || csub == 0) return;
    uint32_t n = 0;
    while (ld_acquire(pflag) == 0u) {
      if (++n >= kFlagPolls) { atomicOr(a.st, ST_TIMEOUT); break; }
      if (n > 64) __nanosleep(32);
    }
    fetch_hin();
  };

  // this row's dt is loaded first so its latency overlaps the readout loads below
  const float dt_row = (half == 0 && row < L) ? a.dt[(size_t)(row0 + row) * d.H + h] : 0.f;

  // C~ rows = sum of the readout slots.  The first slot comes by TMA into CT (issued above with slot 0's
  // keys and values); the others are loaded coalesced (16 lanes per 256-byte row, warp w covers rows
  // 16w .. 16w + 15) and added to CT in shared memory: two slots as one fp16 pair add (the correctly
  // rounded sum), after slot 0's decay-scaled values so that the loads' latency overlaps that work; more
  // slots in fp32, rounded once.
  const int hl = lane >> 4, c16 = lane & 15;
  auto ct_chunk = [&](int u) { const int r = 16 * warp + 2 * u + hl; return CT + (c16 >> 3) * kBlk + tc::sw128_chunk(r, c16 & 7); };
  auto load8 = [&](int j, uint4 (&dst)[8]) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = 16 * warp + 2 * u + hl;
      dst[u] = make_uint4(0u, 0u, 0u, 0u);
      if (r < L)
        dst[u] = __ldg(reinterpret_cast<const uint4*>(a.cpi + ((size_t)(row0 + r) * d.k + j) * d.GN + (size_t)g * N +
                                                      c16 * 8));
    }
  };
  uint4 cq[8];  // the second read slot (two read slots)
  bool c_ok = true;
  if (a.read_slots == 2) {
    load8(a.read_slot0 + 1, cq);
  } else if (a.read_slots >= 3) {
    float acc[8][8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[u][e] = 0.f;
    for (int j = a.read_slot0 + 1; j < a.read_slot0 + a.read_slots; ++j) {
      load8(j, cq);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const __half2* hq = reinterpret_cast<const __half2*>(&cq[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(hq[e]);
          acc[u][2 * e] += f.x;
          acc[u][2 * e + 1] += f.y;
        }
      }
    }
    c_ok = tc::mbar_wait(fullC, 0, &never);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      uint4* dst = reinterpret_cast<uint4*>(ct_chunk(u));
      uint4 v = *dst;
      __half2* hv2 = reinterpret_cast<__half2*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(hv2[e]);
        hv2[e] = __floats2half2_rn(f.x + acc[u][2 * e], f.y + acc[u][2 * e + 1]);
      }
      *dst = v;
    }
  }
  // C~ complete in CT (called by every thread before the first product that reads CT)
  auto finish_ct = [&]() {
    if (a.read_slots >= 3) return;
    c_ok = tc::mbar_wait(fullC, 0, &never) && c_ok;
    if (a.read_slots == 2) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        uint4* dst = reinterpret_cast<uint4*>(ct_chunk(u));
        uint4 v = *dst;
        __half2* x = reinterpret_cast<__half2*>(&v);
        const __half2* y = reinterpret_cast<const __half2*>(&cq[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = __hadd2(x[e], y[e]);
        *dst = v;
      }
    }
  };

  // cumulative log-decay of the sub-chunk (inclusive scan over the 128 rows)
  float v = 0.f;
  if (half == 0) {
    v = dt_row * a.A[h];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane == 31) wsum[warp] = v;
  }
  tc::fence_proxy_async();
  __syncthreads();
  if (half == 0) {
    for (int w = 0; w < warp; ++w) v += wsum[w];
    cs_s[row] = v;
  }
  __syncthreads();
  const float my_cs = cs_s[row], cs_end = cs_s[L - 1];
  // decay factorisation over 32-key blocks: exp(cs_t - cs_s) = exp(cs_t - cs_{32b}) * exp(cs_{32b} - cs_s)
  if (half == 0) fs_s[row] = expf(cs_s[row & ~31] - my_cs);
  const float dec_end = row < L ? expf(cs_end - my_cs) : 0.f;
  __syncthreads();

  bool ok = true;
  uint32_t done_phase = 0;
  const uint32_t ct = tc::smem_u32(CT), bp = tc::smem_u32(BP);
  // slot i's values sit in one of the two value buffers and its decay-scaled copy goes to the other, so
  // slot i + 1's values can be loaded into this copy's buffer once the end-state product has read it
  auto value_buf = [&](int i) { return (i & 1) ? PM : XS; };
  auto scaled_buf = [&](int i) { return (i & 1) ? XS : PM; };
  // wait for slot i's keys and values, scale the values by the decay to the sub-chunk end and issue the
  // end-state product Sc += Bpi_i^T (decay_end * Xs_i)
  auto begin_slot = [&](int i) -> bool {
    const uint32_t par = (uint32_t)(i & 1);
    bool w = tc::mbar_wait(fullX, par, &never) && tc::mbar_wait(fullB, par, &never);
    if (!__syncthreads_and(w)) return false;
    uint8_t* XV = value_buf(i);
    uint8_t* DXV = scaled_buf(i);
    if (tid == 0 && i + 1 == nk) peek_hin();
#pragma unroll
    for (int pb = 0; pb < PB; ++pb) {
#pragma unroll
      for (int c = 4 * half; c < 4 * half + 4; ++c) {
        const uint32_t off = pb * kBlk + tc::sw128_chunk(row, c);
        uint4 q = *reinterpret_cast<const uint4*>(XV + off);
        __half2* hq = reinterpret_cast<__half2*>(&q);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(hq[e]);
          hq[e] = __floats2half2_rn(f.x * dec_end, f.y * dec_end);
        }
        *reinterpret_cast<uint4*>(DXV + off) = q;
      }
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0) {
      const uint32_t dx = tc::smem_u32(DXV);
#pragma unroll
      for (int kk = 0; kk < SUB / 16; ++kk) {
        tc::mma_f16(tmem + COL_SC, tc::sdesc_mnmajor_sw128(bp + kk * 2048, kBlk),
                    tc::sdesc_mnmajor_sw128(dx + kk * 2048, kBlk), ID_SC, (i > 0) || (kk > 0));
      }
    }
    return true;
  };
  // slot 0's end-state product runs while C~ is completed (outside the loop, so the registers holding the
  // second read slot are free in it)
  ok = begin_slot(0);
  if (ok) {
    finish_ct();
    tc::fence_proxy_async();
    if (!__syncthreads_and(c_ok)) {
      ok = false;
      if (tid == 0) {  // the end-state product is in flight: let it finish before TMEM is freed
        tc::mma_commit(done);
        tc::mbar_wait(done, done_phase, &never);
      }
    }
  }
  for (int i = 0; i < nk && ok; ++i) {
    if (i > 0 && !begin_slot(i)) { ok = false; break; }
    uint8_t* XV = value_buf(i);
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < N / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kBlk + (kk & 3) * 32;
        tc::mma_f16(tmem + COL_S, tc::sdesc_kmajor_sw128(ct + off), tc::sdesc_kmajor_sw128(bp + off), ID_S, kk > 0);
      }
      tc::mma_commit(done);
    }
    ok = tc::mbar_wait(done, done_phase, &never);
    done_phase ^= 1u;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    tc::fence_after_sync();
    if (tid == 0 && i + 1 < nk) {  // Bpi_i and the decay-scaled Xs_i are no longer read
      issue_b(i + 1);
      issue_x(i + 1);
    }
    if (tid == 0 && i + 1 == nk) peek_hin();  // the Bpi region is free for good
    // masked, decayed scores of this thread's 64 keys (32-key blocks kb = 2 half and 2 half + 1, whose decays
    // share one factor exp(cs_t - cs_{32b}) per block), packed to fp16 pairs and stored back into TMEM over
    // the first 32 of the same 64 S columns (no other thread reads those), where the next product takes
    // them as its A operand
    {
      uint32_t pk0[16], pk1[16];
      auto pack = [&](int kb, uint32_t (&pk)[16]) {
        uint32_t r[32];
        tc::tmem_ld_32x32b_x32(tmem + lane_base + COL_S + 32 * kb, r);
        const float et = (32 * kb <= row && row < L) ? expf(my_cs - cs_s[32 * kb]) : 0.f;
        float fs[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) fs[e] = et * fs_s[32 * kb + e];
        tc::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int s0 = 32 * kb + 2 * e;
          const float f0 = s0 <= row ? u2f(r[2 * e]) * fs[2 * e] : 0.f;
          const float f1 = s0 + 1 <= row ? u2f(r[2 * e + 1]) * fs[2 * e + 1] : 0.f;
          pk[e] = pack_half2(f0, f1);
        }
      };
      pack(2 * half, pk0);
      pack(2 * half + 1, pk1);
      tc::tmem_st_32x32b_x16(tmem + lane_base + COL_S + 64 * half, pk0);
      tc::tmem_st_32x32b_x16(tmem + lane_base + COL_S + 64 * half + 16, pk1);
      tc::tmem_st_wait();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    // With P = 64 the last slot's Y product runs under the state hand-off that follows (which touches only
    // the Bpi region, TMEM's end-state columns and global memory); the readout product's commit covers it.
    const bool defer = P == 64 && i + 1 == nk;
    if (tid == 0) {
      const uint32_t xs = tc::smem_u32(XV);
#pragma unroll
      for (int kk = 0; kk < SUB / 16; ++kk)
        tc::mma_f16_tmem_a(tmem + COL_Y, tmem + COL_S + 8 * kk + (kk >= 4 ? 32 : 0),
                           tc::sdesc_mnmajor_sw128(xs + kk * 2048, kBlk), ID_Y, (i > 0) || (kk > 0));
      if (!defer) tc::mma_commit(done);
    }
    if (defer) break;
    ok = tc::mbar_wait(done, done_phase, &never);
    done_phase ^= 1u;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    tc::fence_after_sync();
    if (tid == 0 && i + 1 == nk) peek_hin();
  }

  if (ok) {
    // ---------------------------------------------------------------- state hand-off
    const size_t NP = NPs;
    if (tid == 0 && csub > 0) {
      if (kEarlyFetch) {
        wait_fetch_hin();
      } else {
        uint32_t n = 0;
        while (ld_acquire(pflag) == 0u && n < kFlagPolls) {
          if (n > 64) __nanosleep(32);
          ++n;
        }
        if (n == kFlagPolls) atomicOr(a.st, ST_TIMEOUT);
      }
    }
    bool hok = true;
    if (kEarlyFetch && csub > 0) hok = tc::mbar_wait(hbar, 0, &never);
    hok = __syncthreads_and(hok);
    if (!hok && tid == 0) atomicOr(a.st, ST_TIMEOUT);  // continues with a zero state; the result is flagged
    const bool hin_shared = kEarlyFetch && csub > 0;
    const float* hin = csub > 0 ? (hin_shared ? (hok ? reinterpret_cast<const float*>(BP) : nullptr) : hprev)
                                : (a.init ? a.init + (size_t)bh * NP : nullptr);
    float* hout = a.exch + ((size_t)bh * a.nsub + csub) * NP;
    const float dend = expf(cs_end);
    const size_t rbase = (size_t)row * P + half * PH;
    // this thread's half row of H_in (kept for the fp16 split below) and H_out = exp(cs_end) H_in + Sc
    // exchanged states are stored thread-major (float4 U of thread tid at (U * kThreads + tid) * 4) so the
    // stores coalesce and the reads from shared memory are conflict-free; the initial state is [N][P]
    auto xidx = [&](int U) { return ((size_t)U * kThreads + tid) * 4; };
    const bool hin_canon = csub == 0;
    float4 hv[PH / 4];
#pragma unroll
    for (int u = 0; u < PH / 4; ++u)
      hv[u] = !hin ? make_float4(0.f, 0.f, 0.f, 0.f)
                   : (hin_shared ? *reinterpret_cast<const float4*>(hin + xidx(u))
                                 : __ldcg(reinterpret_cast<const float4*>(hin + (hin_canon ? rbase + 4 * u : xidx(u)))));
#pragma unroll
    for (int q = 0; q < PH / 32; ++q) {
      uint32_t r[32];
      tc::tmem_ld_32x32b_x32(tmem + lane_base + COL_SC + half * PH + 32 * q, r);
      tc::tmem_ld_wait();
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 x = hv[8 * q + u];
        const float4 o = make_float4(fmaf(dend, x.x, u2f(r[4 * u])), fmaf(dend, x.y, u2f(r[4 * u + 1])),
                                     fmaf(dend, x.z, u2f(r[4 * u + 2])), fmaf(dend, x.w, u2f(r[4 * u + 3])));
        __stcg(reinterpret_cast<float4*>(hout + xidx(8 * q + u)), o);
      }
    }
    // every thread's H_out stores are ordered before the barrier; thread 0's release store at device scope
    // is cumulative over them, so a consumer that acquires the flag sees the whole state
    __syncthreads();
    if (tid == 0) st_release(a.flags + (size_t)bh * a.nsub + csub, 1u);
    // off the hand-off chain: requested states, and the fp16 hi/lo split of H_in for the readout product
    const bool last = t0 + L == d.T;
    const bool chunk_start = a.chunk_states && (t0 % d.Q) == 0;
    float* cst = chunk_start ? a.chunk_states + (((size_t)b * d.H + h) * d.nc + t0 / d.Q) * NP : nullptr;
    float* fin = (last && a.final_state) ? a.final_state + (size_t)bh * NP : nullptr;
    uint8_t* HH = BP;  // Bpi_j and Xs_j are consumed
    uint8_t* HL = BP + PB * kBlk;
    bool range_bad = false;
#pragma unroll
    for (int u = 0; u < PH / 4; ++u) {
      if (cst) *reinterpret_cast<float4*>(cst + rbase + 4 * u) = hv[u];
      if (fin) *reinterpret_cast<float4*>(fin + rbase + 4 * u) = __ldcg(reinterpret_cast<const float4*>(hout + xidx(u)));
    }
#pragma unroll
    for (int c = 0; c < PH / 8; ++c) {
      float hp[8], hi[8], lo[8];
      hp[0] = hv[2 * c].x; hp[1] = hv[2 * c].y; hp[2] = hv[2 * c].z; hp[3] = hv[2 * c].w;
      hp[4] = hv[2 * c + 1].x; hp[5] = hv[2 * c + 1].y; hp[6] = hv[2 * c + 1].z; hp[7] = hv[2 * c + 1].w;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        hi[e] = __half2float(__float2half_rn(hp[e]));
        lo[e] = hp[e] - hi[e];
        range_bad |= !(fabsf(hp[e]) <= kF16Max);
      }
      const int p0 = half * PH + 8 * c;
      const uint32_t off = (p0 >> 6) * kBlk + tc::sw128_chunk(row, (p0 & 63) >> 3);
      uint4 oh, ol;
      oh.x = pack_half2(hi[0], hi[1]); oh.y = pack_half2(hi[2], hi[3]);
      oh.z = pack_half2(hi[4], hi[5]); oh.w = pack_half2(hi[6], hi[7]);
      ol.x = pack_half2(lo[0], lo[1]); ol.y = pack_half2(lo[2], lo[3]);
      ol.z = pack_half2(lo[4], lo[5]); ol.w = pack_half2(lo[6], lo[7]);
      *reinterpret_cast<uint4*>(HH + off) = oh;
      *reinterpret_cast<uint4*>(HL + off) = ol;
    }
    if (range_bad) atomicOr(a.st, ST_RANGE);
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0) {
      const uint32_t ct = tc::smem_u32(CT), hh = tc::smem_u32(HH), hl2 = tc::smem_u32(HL);
#pragma unroll
      for (int kk = 0; kk < N / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kBlk + (kk & 3) * 32;
        tc::mma_f16(tmem + COL_S, tc::sdesc_kmajor_sw128(ct + off), tc::sdesc_mnmajor_sw128(hh + kk * 2048, kBlk),
                    ID_Y, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < N / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kBlk + (kk & 3) * 32;
        tc::mma_f16(tmem + COL_S, tc::sdesc_kmajor_sw128(ct + off), tc::sdesc_mnmajor_sw128(hl2 + kk * 2048, kBlk),
                    ID_Y, 1);
      }
      tc::mma_commit(done);
    }
    ok = tc::mbar_wait(done, done_phase, &never);
    done_phase ^= 1u;
    if (__syncthreads_and(ok)) {
      tc::fence_after_sync();
      // ---------------------------------------------------------------- output rows (this thread's half)
      const float eq = expf(my_cs);
      const bool valid = row < L;
      const size_t orow = (size_t)(row0 + row) * d.HP + (size_t)h * P + half * PH;
#pragma unroll
      for (int q = 0; q < PH / 32; ++q) {
        uint32_t ry[32], ri[32];
        tc::tmem_ld_32x32b_x32(tmem + lane_base + COL_Y + half * PH + 32 * q, ry);
        tc::tmem_ld_32x32b_x32(tmem + lane_base + COL_S + half * PH + 32 * q, ri);
        tc::tmem_ld_wait();
        if (!valid) continue;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = fmaf(eq, u2f(ri[8 * c + e]), u2f(ry[8 * c + e]));
          const size_t o = orow + 32 * q + 8 * c;
          if (a.accumulate_y) {
            if (!a.first_pass) {
#pragma unroll
              for (int e = 0; e < 8; ++e) f[e] += a.ysum[o + e];
            }
            if (!a.last_pass) {
#pragma unroll
              for (int e = 0; e < 8; ++e) a.ysum[o + e] = f[e];
              continue;
            }
          }
          uint4 ov;
          __nv_bfloat162 b0 = __floats2bfloat162_rn(f[0], f[1]), b1 = __floats2bfloat162_rn(f[2], f[3]);
          __nv_bfloat162 b2 = __floats2bfloat162_rn(f[4], f[5]), b3 = __floats2bfloat162_rn(f[6], f[7]);
          ov.x = *reinterpret_cast<uint32_t*>(&b0); ov.y = *reinterpret_cast<uint32_t*>(&b1);
          ov.z = *reinterpret_cast<uint32_t*>(&b2); ov.w = *reinterpret_cast<uint32_t*>(&b3);
          *reinterpret_cast<uint4*>(a.y + o) = ov;
        }
      }
    }
  }
  if (!ok && tid == 0) {
    atomicOr(a.st, ST_TIMEOUT);
    st_release(a.flags + (size_t)bh * a.nsub + csub, 1u);  // successors must not wait on a CTA that gave up
  }
  // no copy may still be landing in shared memory when the CTA exits
  if (tid == 0) {
    if (issuedB > 0) tc::mbar_wait(fullB, (uint32_t)((issuedB - 1) & 1), &never);
    if (issuedX > 0) tc::mbar_wait(fullX, (uint32_t)((issuedX - 1) & 1), &never);
    if (h_issued) tc::mbar_wait(hbar, 0, &never);
    tc::mbar_wait(fullC, 0, &never);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

bool scan_tc_supported(const Dims& d) {
  return d.dtype == SWIMBA_BF16 && d.N == 128 && (d.P == 64 || d.P == 128);
}

int scan_tc_subchunks(const Dims& d) { return ceil_div(d.T, SUB); }

// lb: zeroed by the caller (ticket counter at lb[0], flags at lb + 64); exch: [B*H][nsub] states of N*P
// fp32, each stored thread-major (see the hand-off).
cudaError_t launch_scan_tc(const Dims& d, const ScanArgs& s, unsigned* lb, float* exch, unsigned* st,
                           cudaStream_t stream) {
  CUtensorMap tb, tx;
  if (!encode_tmap_3d_slot(&tb, s.bpi, SWIMBA_F16, (uint64_t)d.GN, (uint64_t)d.k, (uint64_t)d.M, 64, SUB))
    return cudaErrorInvalidValue;
  if (!encode_tmap_3d_slot(&tx, s.xs, SWIMBA_F16, (uint64_t)d.HP, (uint64_t)d.k, (uint64_t)d.M, 64, SUB))
    return cudaErrorInvalidValue;
  CUtensorMap tc3;
  if (!encode_tmap_3d_slot(&tc3, s.cpi, SWIMBA_F16, (uint64_t)d.GN, (uint64_t)d.k, (uint64_t)d.M, 64, SUB))
    return cudaErrorInvalidValue;
  TcScanArgs a{};
  a.d = d; a.dt = s.dt; a.A = s.A; a.init = s.init; a.cpi = (const __half*)s.cpi; a.y = (__nv_bfloat16*)s.y;
  a.final_state = s.final_state; a.chunk_states = s.chunk_states; a.exch = exch; a.flags = lb + 64; a.ticket = lb;
  a.st = st; a.ysum = s.ysum; a.nsub = scan_tc_subchunks(d);
  a.key_slot0 = s.key_slot0; a.key_slots = s.key_slots; a.read_slot0 = s.read_slot0; a.read_slots = s.read_slots;
  a.accumulate_y = s.accumulate_y; a.first_pass = s.first_pass; a.last_pass = s.last_pass;
  const int grid = d.Bsz * d.H * a.nsub;
  cudaError_t e;
  if (d.P == 64) {
    const size_t sm = ScanSmem<64>::bytes();
    e = set_max_dynamic_smem((const void*)scan_tc_kernel<64>, sm);
    if (e != cudaSuccess) return e;
    e = launch_dependent(scan_tc_kernel<64>, dim3(grid), dim3(kThreads), sm, stream, 1, tb, tx, tc3, a);
    if (e != cudaSuccess) return e;
  } else {
    const size_t sm = ScanSmem<128>::bytes();
    e = set_max_dynamic_smem((const void*)scan_tc_kernel<128>, sm);
    if (e != cudaSuccess) return e;
    e = launch_dependent(scan_tc_kernel<128>, dim3(grid), dim3(kThreads), sm, stream, 1, tb, tx, tc3, a);
    if (e != cudaSuccess) return e;
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swimba
