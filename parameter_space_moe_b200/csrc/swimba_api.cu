// C ABI of libswimba: argument validation, workspace planning and the launch sequence of each entry
// point.  Every entry point validates before launching anything and launches asynchronously on the
// caller's stream; nothing here allocates device memory.
#include <atomic>
#include <map>
#include <mutex>

#include "common.cuh"

namespace swimba {

// Sticky device status word (bits ST_*), one per device; read and cleared by
// swimba_check_device_status.  Host code only ever uses its device address (device_status()).
__device__ unsigned g_status_word;

// The address is looked up once per device and kept for the life of the process (a device reset between
// calls is not supported: it would reload the module and leave the kept address stale).
unsigned* device_status() {
  static std::mutex mu;
  static unsigned* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    addr[dev] = (unsigned*)p;
  }
  return addr[dev];
}

// ---------------------------------------------------------------------------------------------
// Launch counter and optional per-stage event timing (see swimba_profile_enable).
static std::atomic<long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

cudaError_t set_max_dynamic_smem(const void* kernel, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, size_t> granted;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  size_t& g = granted[{dev, kernel}];
  if (bytes <= g) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) g = bytes;
  return e;
}

struct Profiler {
  static constexpr int kMax = 16;
  std::mutex mu;
  bool on = false, created = false;
  int n = 0;
  const char* name[kMax];
  cudaEvent_t ev[kMax + 1];
};
static Profiler g_prof;

static void prof_begin(cudaStream_t s) {
  if (!g_prof.on) return;
  g_prof.n = 0;
  cudaEventRecord(g_prof.ev[0], s);
}
static void prof_mark(cudaStream_t s, const char* stage) {
  if (!g_prof.on || g_prof.n >= Profiler::kMax) return;
  g_prof.name[g_prof.n] = stage;
  cudaEventRecord(g_prof.ev[++g_prof.n], s);
}

size_t elem_bytes(int dtype) { return dtype == SWIMBA_F32 ? 4 : 2; }
int stream_dtype_of(int dtype) { return dtype == SWIMBA_F32 ? SWIMBA_F32 : SWIMBA_F16; }

WsPlan plan_workspace(const Dims& d) {
  WsPlan p{};
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  const size_t Mk = (size_t)d.M * d.k;
  const size_t sb = elem_bytes(stream_dtype_of(d.dtype));
  // chunk states: per Q-token chunk for the CUDA-core scan, per 64-token sub-chunk for the scan gradients
  const size_t nst = (size_t)scan_bwd_subchunks(d) > (size_t)d.nc ? (size_t)scan_bwd_subchunks(d) : (size_t)d.nc;
  const size_t states = (size_t)d.Bsz * d.H * nst * d.N * d.P * 4;
  p.status = take(256);
  p.topk_idx = take(Mk * 4);
  p.topk_w = take(Mk * 4);
  p.dt = take((size_t)d.M * d.H * 4);
  p.dA = take((size_t)d.M * d.H * 4);
  p.ones = take((size_t)d.H * 4);
  p.dcounts = take((size_t)dispatch_tiles(d) * d.E * 4);
  const size_t nsub = (size_t)scan_tc_subchunks(d);
  p.lb_bytes = 256 + (size_t)d.Bsz * d.H * nsub * 4;
  p.lb = take(p.lb_bytes);  // directly after dcounts: run_front clears both with one kernel
  p.dbase = take((size_t)dispatch_tiles(d) * d.E * 4);
  p.offsets = take((size_t)(d.E + 1) * 4);
  p.perm = take(Mk * 4);
  p.rowmeta = take(Mk * 8);
  p.tiles = take((size_t)max_row_tiles(d) * 8);
  p.ntiles = take(4);
  p.xsorted = take(Mk * d.D * elem_bytes(d.dtype));
  p.bpi = take(Mk * d.GN * sb);
  p.xs = take(Mk * d.HP * sb);
  p.cpi = take(Mk * d.GN * sb);
  p.yintra = take((size_t)d.M * d.HP * 4);
  p.ysum = take((size_t)d.M * d.HP * 4);
  p.schunk = take(states);
  p.hstart = take(states);
  p.cslast = take((size_t)d.Bsz * d.H * nst * 4);
  p.exch = take((size_t)d.Bsz * d.H * nsub * d.N * d.P * 4);
  p.total = o;
  return p;
}

static bool pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

swimba_status make_dims(const swimba_dims* in, Dims* d) {
  if (!in) return SWIMBA_ERR_INVALID_ARG;
  const swimba_dims& s = *in;
  if (s.batch < 1 || s.seqlen < 1 || s.d_model < 1 || s.nheads < 1 || s.headdim < 1 || s.dstate < 1 ||
      s.ngroups < 1 || s.n_experts < 1 || s.top_k < 1 || s.chunk < 1)
    return SWIMBA_ERR_INVALID_ARG;
  if (s.dtype != SWIMBA_F32 && s.dtype != SWIMBA_BF16) return SWIMBA_ERR_INVALID_ARG;
  if (s.top_k > s.n_experts || s.nheads % s.ngroups != 0) return SWIMBA_ERR_INVALID_ARG;
  if (!pow2_in(s.headdim, 16, 128) || !pow2_in(s.dstate, 16, 128) || !pow2_in(s.chunk, 64, 256))
    return SWIMBA_ERR_UNSUPPORTED;
  if (s.top_k > 8 || s.n_experts > 64) return SWIMBA_ERR_UNSUPPORTED;
  if (s.d_model % (s.dtype == SWIMBA_BF16 ? 64 : 8) != 0) return SWIMBA_ERR_UNSUPPORTED;
  const long long M = (long long)s.batch * s.seqlen;
  const long long HP = (long long)s.nheads * s.headdim, GN = (long long)s.ngroups * s.dstate;
  if (M * s.top_k >= (1LL << 30) || HP + 2 * GN >= (1LL << 24) || M * HP >= (1LL << 40))
    return SWIMBA_ERR_UNSUPPORTED;
  d->Bsz = s.batch; d->T = s.seqlen; d->D = s.d_model; d->H = s.nheads; d->P = s.headdim; d->N = s.dstate;
  d->G = s.ngroups; d->E = s.n_experts; d->k = s.top_k; d->Q = s.chunk; d->dtype = s.dtype;
  d->M = (int)M; d->HP = (int)HP; d->GN = (int)GN; d->We = (int)(HP + 2 * GN);
  d->nc = ceil_div(s.seqlen, s.chunk); d->hpg = s.nheads / s.ngroups;
  return SWIMBA_OK;
}

static bool aligned(const void* p) { return ((uintptr_t)p & 15u) == 0; }
static bool ok_ptr(const void* p) { return p && aligned(p); }
static bool ok_opt(const void* p) { return !p || aligned(p); }

static swimba_status check_weights(const swimba_weights* w, bool need_router, bool need_exp) {
  if (!w) return SWIMBA_ERR_INVALID_ARG;
  if (need_router && (!ok_ptr(w->w_router) || !ok_ptr(w->w_dt) || !w->b_dt || (!w->A && !w->A_exp)))
    return SWIMBA_ERR_INVALID_ARG;
  if (need_exp && !ok_ptr(w->w_exp)) return SWIMBA_ERR_INVALID_ARG;
  return SWIMBA_OK;
}

static swimba_status check_ws(const Dims& d, const void* ws, size_t bytes) {
  if (!ws || !aligned(ws) || bytes < plan_workspace(d).total) return SWIMBA_ERR_WORKSPACE;
  return SWIMBA_OK;
}

static swimba_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SWIMBA_OK : SWIMBA_ERR_CUDA; }

#define SW_TRY(x)                                   \
  do {                                              \
    swimba_status s_ = (x);                         \
    if (s_ != SWIMBA_OK) return s_;                 \
  } while (0)
#define SW_CUDA(x)                                  \
  do {                                              \
    cudaError_t e_ = (x);                           \
    if (e_ != cudaSuccess) return SWIMBA_ERR_CUDA;  \
  } while (0)

// Expert projections of the dispatched rows (after launch_dispatch): bf16 layers gather X into expert
// order and run the tensor-core GEMM; the fp32 layer runs the CUDA-core GEMM.
static swimba_status run_proj(const Dims& d, const void* X, const void* w_exp, char* ws, const WsPlan& p,
                              const float* wts, int mode, void* bpi, void* xs, void* cpi, float* Z, unsigned* st,
                              cudaStream_t s, bool gathered = false) {
  const int32_t* offsets = (const int32_t*)(ws + p.offsets);
  const int32_t* perm = (const int32_t*)(ws + p.perm);
  const int32_t* tiles = (const int32_t*)(ws + p.tiles);
  const int32_t* ntiles = (const int32_t*)(ws + p.ntiles);
  if (d.dtype == SWIMBA_BF16) {
    if (!gathered) {
      SW_CUDA(launch_gather_rows(d, X, perm, ws + p.xsorted, s));
      prof_mark(s, "gather");
    }
    SW_CUDA(launch_proj_tc(d, ws + p.xsorted, w_exp, (const int2*)(ws + p.rowmeta), tiles, ntiles, offsets, mode, bpi,
                           xs, cpi, Z, st, s));
  } else {
    SW_CUDA(launch_proj_simt(d, X, w_exp, perm, tiles, ntiles, offsets, wts, mode, bpi, xs, cpi, Z, st, s));
  }
  prof_mark(s, "expert_proj_mix");
  return SWIMBA_OK;
}

// Router + dispatch + projection with the fused mix, into the workspace's streams (mode 4: also the raw B
// and C columns of z into Z).
static swimba_status run_front(const Dims& d, const void* X, const swimba_weights* w, char* ws, const WsPlan& p,
                               int32_t* idx, float* wts, int mode, unsigned* st, cudaStream_t s,
                               float* Z = nullptr) {
  float* dt = (float*)(ws + p.dt);
  // one small kernel clears the router's per-tile counts and the scan's hand-off flags (adjacent regions);
  // the router's prologue and loads overlap it
  SW_CUDA(launch_zero_u32((unsigned*)(ws + p.dcounts), (p.lb + p.lb_bytes - p.dcounts) / 4, s));
  int32_t* counts = (int32_t*)(ws + p.dcounts);
  SW_CUDA(launch_router(d, X, *w, idx, wts, dt, counts, st, s, /*after_zero=*/true));
  prof_mark(s, "router");
  int32_t* offsets = (int32_t*)(ws + p.offsets);
  int32_t* perm = (int32_t*)(ws + p.perm);
  const bool fused_gather = d.dtype == SWIMBA_BF16;
  if (fused_gather) {
    SW_CUDA(launch_dispatch_gather(d, idx, counts, p, ws, offsets, perm, wts, X, s));
    prof_mark(s, "dispatch_gather");
  } else {
    SW_CUDA(launch_dispatch_fused(d, idx, counts, p, ws, offsets, perm, wts, s));
    prof_mark(s, "dispatch");
  }
  SW_TRY(run_proj(d, X, w->w_exp, ws, p, wts, mode, ws + p.bpi, ws + p.xs, ws + p.cpi, Z, st, s, fused_gather));
  return SWIMBA_OK;
}

// The chunked scan: tensor-core kernel for the shapes it covers, CUDA-core kernels otherwise (the
// fp32 layer, N != 128, P not in {64, 128}, or per-chunk states requested at chunk 64).
static swimba_status run_scan(const Dims& d, const ScanArgs& a, char* ws, const WsPlan& p, cudaStream_t s,
                              bool lb_clear = false) {
  if (scan_tc_supported(d) && !(a.chunk_states && d.Q < 128)) {
    if (!lb_clear) SW_CUDA(cudaMemsetAsync(ws + p.lb, 0, p.lb_bytes, s));
    SW_CUDA(launch_scan_tc(d, a, (unsigned*)(ws + p.lb), (float*)(ws + p.exch), device_status(), s));
  } else {
    SW_CUDA(launch_scan_simt(d, a, s));
  }
  return SWIMBA_OK;
}

// Expert-mixed transition (weights.A_exp given): dA = dt * A~ per token and head and A = 1, which the scan
// and the decode step read in place of dt and the shared A (dt * 1 is exact).
static swimba_status run_mixed_a(const Dims& d, const swimba_weights* w, const int32_t* idx, const float* wts,
                                 char* ws, const WsPlan& p, const float** dt, const float** A, cudaStream_t s) {
  if (!w->A_exp) return SWIMBA_OK;
  float* dA = (float*)(ws + p.dA);
  float* ones = (float*)(ws + p.ones);
  SW_CUDA(launch_mixed_a(d, idx, wts, w->A_exp, *dt, dA, ones, device_status(), s));
  prof_mark(s, "mixed_A");
  *dt = dA;
  *A = ones;
  return SWIMBA_OK;
}

static ScanArgs mixed_scan_args(const Dims& d, char* ws, const WsPlan& p, const void* bpi, const void* xs,
                                const void* cpi, const float* dt, const float* A, const float* init, void* y,
                                float* final_state, float* chunk_states) {
  ScanArgs a{};
  a.bpi = bpi; a.xs = xs; a.cpi = cpi; a.dt = dt; a.A = A; a.init = init; a.y = y;
  a.final_state = final_state;
  a.hstart = chunk_states ? chunk_states : (float*)(ws + p.hstart);
  a.chunk_states = chunk_states;
  a.schunk = (float*)(ws + p.schunk); a.cslast = (float*)(ws + p.cslast);
  a.yacc = (float*)(ws + p.yintra); a.ysum = (float*)(ws + p.ysum);
  a.key_slot0 = 0; a.key_slots = d.k; a.read_slot0 = 0; a.read_slots = d.k;
  a.accumulate_y = false;
  return a;
}

}  // namespace swimba

using namespace swimba;

extern "C" {

size_t swimba_workspace_size(const swimba_dims* dims) {
  Dims d;
  if (make_dims(dims, &d) != SWIMBA_OK) return 0;
  return plan_workspace(d).total;
}

int swimba_stream_dtype(const swimba_dims* dims) {
  Dims d;
  if (make_dims(dims, &d) != SWIMBA_OK) return -1;
  return stream_dtype_of(d.dtype);
}

swimba_status swimba_router_topk(const swimba_dims* dims, const void* X, const swimba_weights* w,
                                 int32_t* topk_idx, float* topk_w, float* dt, void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  SW_TRY(check_weights(w, true, false));
  if (!ok_ptr(X) || !ok_ptr(topk_idx) || !ok_ptr(topk_w) || !ok_ptr(dt)) return SWIMBA_ERR_INVALID_ARG;
  unsigned* st = device_status();
  if (!st) return SWIMBA_ERR_CUDA;
  return cuda_status(launch_router(d, X, *w, topk_idx, topk_w, dt, nullptr, st, (cudaStream_t)stream));
}

swimba_status swimba_dispatch(const swimba_dims* dims, const int32_t* topk_idx, int32_t* expert_offsets,
                              int32_t* perm, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  if (!ok_ptr(topk_idx) || !ok_ptr(expert_offsets) || !ok_ptr(perm)) return SWIMBA_ERR_INVALID_ARG;
  SW_TRY(check_ws(d, ws, ws_bytes));
  WsPlan p = plan_workspace(d);
  unsigned* st = device_status();
  if (!st) return SWIMBA_ERR_CUDA;
  return cuda_status(
      launch_dispatch(d, topk_idx, p, (char*)ws, expert_offsets, perm, nullptr, nullptr, st, (cudaStream_t)stream));
}

swimba_status swimba_expert_proj(const swimba_dims* dims, const void* X, const swimba_weights* w,
                                 const int32_t* topk_idx, float* Z, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  SW_TRY(check_weights(w, false, true));
  if (!ok_ptr(X) || !ok_ptr(topk_idx) || !ok_ptr(Z)) return SWIMBA_ERR_INVALID_ARG;
  SW_TRY(check_ws(d, ws, ws_bytes));
  WsPlan p = plan_workspace(d);
  char* b = (char*)ws;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t* offsets = (int32_t*)(b + p.offsets);
  int32_t* perm = (int32_t*)(b + p.perm);
  unsigned* st = device_status();
  if (!st) return SWIMBA_ERR_CUDA;
  SW_CUDA(launch_dispatch(d, topk_idx, p, b, offsets, perm, (int2*)(b + p.rowmeta), nullptr, st, s));
  return run_proj(d, X, w->w_exp, b, p, nullptr, 2, nullptr, nullptr, nullptr, Z, st, s);
}

swimba_status swimba_mix(const swimba_dims* dims, const float* Z, const float* topk_w, int32_t flags, void* Bpi,
                         void* Xs, void* Cpi, void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  if (!ok_ptr(Z) || !ok_ptr(topk_w) || !ok_ptr(Bpi) || !ok_ptr(Xs) || !ok_ptr(Cpi)) return SWIMBA_ERR_INVALID_ARG;
  if (flags & ~SWIMBA_MIX_UNSCALED_B) return SWIMBA_ERR_INVALID_ARG;
  return cuda_status(launch_mix(d, Z, topk_w, flags, Bpi, Xs, Cpi, device_status(), (cudaStream_t)stream));
}

swimba_status swimba_ssd_scan(const swimba_dims* dims, const void* Bpi, const void* Xs, const void* Cpi,
                              const float* dt, const float* A, const float* init_state, void* y,
                              float* final_state, float* chunk_states, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  if (!ok_ptr(Bpi) || !ok_ptr(Xs) || !ok_ptr(Cpi) || !ok_ptr(dt) || !A || !ok_ptr(y)) return SWIMBA_ERR_INVALID_ARG;
  if (!ok_opt(init_state) || !ok_opt(final_state) || !ok_opt(chunk_states)) return SWIMBA_ERR_INVALID_ARG;
  SW_TRY(check_ws(d, ws, ws_bytes));
  WsPlan p = plan_workspace(d);
  ScanArgs a = mixed_scan_args(d, (char*)ws, p, Bpi, Xs, Cpi, dt, A, init_state, y, final_state, chunk_states);
  cudaStream_t s = (cudaStream_t)stream;
  prof_begin(s);
  SW_TRY(run_scan(d, a, (char*)ws, p, s));
  prof_mark(s, "ssd_scan");
  return SWIMBA_OK;
}

namespace {
__global__ void set_u32_kernel(unsigned* p, unsigned v) { *p = v; }
cudaError_t launch_fill_u32(unsigned* p, unsigned v, cudaStream_t s) {
  set_u32_kernel<<<1, 1, 0, s>>>(p, v);
  count_launches(1);
  return cudaGetLastError();
}
}  // namespace

swimba_status swimba_debug_scan_lost_first_chunk(const swimba_dims* dims, const void* Bpi, const void* Xs,
                                                 const void* Cpi, const float* dt, const float* A, void* y,
                                                 void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  if (!scan_tc_supported(d) || d.T <= 128) return SWIMBA_ERR_UNSUPPORTED;
  if (!ok_ptr(Bpi) || !ok_ptr(Xs) || !ok_ptr(Cpi) || !ok_ptr(dt) || !A || !ok_ptr(y)) return SWIMBA_ERR_INVALID_ARG;
  SW_TRY(check_ws(d, ws, ws_bytes));
  WsPlan p = plan_workspace(d);
  char* b = (char*)ws;
  ScanArgs a = mixed_scan_args(d, b, p, Bpi, Xs, Cpi, dt, A, nullptr, y, nullptr, nullptr);
  cudaStream_t s = (cudaStream_t)stream;
  // flags zeroed, ticket counter past every head's first sub-chunk: nothing ever publishes those flags
  SW_CUDA(cudaMemsetAsync(b + p.lb, 0, p.lb_bytes, s));
  SW_CUDA(launch_fill_u32((unsigned*)(b + p.lb), (unsigned)(d.Bsz * d.H), s));
  SW_CUDA(launch_scan_tc(d, a, (unsigned*)(b + p.lb), (float*)(b + p.exch), device_status(), s));
  return SWIMBA_OK;
}

swimba_status swimba_layer_fwd(const swimba_dims* dims, const void* X, const swimba_weights* w,
                               const float* init_state, void* y, float* final_state, int32_t* topk_idx_out,
                               float* topk_w_out, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  SW_TRY(check_weights(w, true, true));
  if (!ok_ptr(X) || !ok_ptr(y) || !ok_opt(init_state) || !ok_opt(final_state) || !ok_opt(topk_idx_out) ||
      !ok_opt(topk_w_out))
    return SWIMBA_ERR_INVALID_ARG;
  SW_TRY(check_ws(d, ws, ws_bytes));
  WsPlan p = plan_workspace(d);
  char* b = (char*)ws;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t* idx = topk_idx_out ? topk_idx_out : (int32_t*)(b + p.topk_idx);
  float* wts = topk_w_out ? topk_w_out : (float*)(b + p.topk_w);
  prof_begin(s);
  SW_TRY(run_front(d, X, w, b, p, idx, wts, 0, device_status(), s));
  const float *dt = (float*)(b + p.dt), *A = w->A;
  SW_TRY(run_mixed_a(d, w, idx, wts, b, p, &dt, &A, s));
  ScanArgs a = mixed_scan_args(d, b, p, b + p.bpi, b + p.xs, b + p.cpi, dt, A, init_state, y, final_state, nullptr);
  SW_TRY(run_scan(d, a, b, p, s, /*lb_clear=*/true));  // run_front already cleared the hand-off flags
  prof_mark(s, "ssd_scan");
  return SWIMBA_OK;
}

// Copy streams and events of swimba_layer_fwd_host, created once per device.
namespace {
constexpr int kMaxHostChunks = 16;
struct HostPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, in[kMaxHostChunks] = {}, out[kMaxHostChunks] = {}, done = nullptr;
  bool ready = false;
};
cudaError_t host_pipe(HostPipe** out) {
  static std::mutex mu;
  static HostPipe pipes[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  HostPipe& q = pipes[dev];
  if (!q.ready) {
    if ((e = cudaStreamCreateWithFlags(&q.h2d, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&q.d2h, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&q.start, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&q.done, cudaEventDisableTiming)) != cudaSuccess) return e;
    for (int c = 0; c < kMaxHostChunks; ++c) {
      if ((e = cudaEventCreateWithFlags(&q.in[c], cudaEventDisableTiming)) != cudaSuccess) return e;
      if ((e = cudaEventCreateWithFlags(&q.out[c], cudaEventDisableTiming)) != cudaSuccess) return e;
    }
    q.ready = true;
  }
  *out = &q;
  return cudaSuccess;
}
}  // namespace

swimba_status swimba_layer_fwd_host(const swimba_dims* dims, const void* X_host, const swimba_weights* w,
                                    const float* init_state, void* y_host, float* final_state, void* X_dev,
                                    void* y_dev, void* ws, size_t ws_bytes, int chunks, void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  if (!X_host || !y_host || !ok_ptr(X_dev) || !ok_ptr(y_dev) || chunks < 1) return SWIMBA_ERR_INVALID_ARG;
  SW_TRY(check_ws(d, ws, ws_bytes));
  HostPipe* q = nullptr;
  SW_CUDA(host_pipe(&q));
  cudaStream_t s = (cudaStream_t)stream;
  const int want = chunks < kMaxHostChunks ? chunks : kMaxHostChunks;
  const size_t xrow = (size_t)d.D * elem_bytes(d.dtype), yrow = (size_t)d.HP * elem_bytes(d.dtype);
  const size_t state = (size_t)d.H * d.N * d.P;
  // With final_state given the groups are time segments of whole 128-token sub-chunks of every sequence,
  // chained through final_state (segment c starts from segment c - 1's final state): each group keeps all
  // (sequence, head) rows, so the scan's hand-off chains stay short.  Otherwise groups of whole sequences.
  const int max_seg = ceil_div(d.T, 128);
  const bool by_time = want > 1 && final_state != nullptr && max_seg > 1;
  const int nch = by_time ? (want < max_seg ? want : max_seg) : (want < d.Bsz ? want : d.Bsz);
  // the copies start after the work already queued on `stream`
  SW_CUDA(cudaEventRecord(q->start, s));
  SW_CUDA(cudaStreamWaitEvent(q->h2d, q->start, 0));
  SW_CUDA(cudaStreamWaitEvent(q->d2h, q->start, 0));
  for (int c = 0; c < nch; ++c) {
    swimba_dims dc = *dims;
    size_t r0;          // the group's first row in the staging buffers (group-major: [batch][len] of the group)
    size_t h0, len, n;  // host side: n blocks of len rows, block b at row h0 + b * T
    const float* init_c;
    float* fin_c;
    if (by_time) {  // sub-chunk-aligned time segments of every sequence
      const int s0 = (int)((long long)max_seg * c / nch) * 128, s1 = c + 1 == nch ? d.T : (int)((long long)max_seg * (c + 1) / nch) * 128;
      len = (size_t)(s1 - s0);
      n = (size_t)d.Bsz;
      h0 = (size_t)s0;
      r0 = (size_t)d.Bsz * s0;
      dc.seqlen = s1 - s0;
      init_c = c == 0 ? init_state : final_state;
      fin_c = final_state;
    } else {  // groups of whole sequences
      const int b0 = (int)((long long)d.Bsz * c / nch), b1 = (int)((long long)d.Bsz * (c + 1) / nch);
      len = (size_t)(b1 - b0) * d.T;
      n = 1;
      h0 = (size_t)b0 * d.T;
      r0 = h0;
      dc.batch = b1 - b0;
      init_c = init_state ? init_state + (size_t)b0 * state : nullptr;
      fin_c = final_state ? final_state + (size_t)b0 * state : nullptr;
    }
    const size_t hstride = n > 1 ? (size_t)d.T : len;  // host rows from one block to the next
    SW_CUDA(cudaMemcpy2DAsync((char*)X_dev + r0 * xrow, len * xrow, (const char*)X_host + h0 * xrow, hstride * xrow,
                              len * xrow, n, cudaMemcpyHostToDevice, q->h2d));
    SW_CUDA(cudaEventRecord(q->in[c], q->h2d));
    SW_CUDA(cudaStreamWaitEvent(s, q->in[c], 0));
    SW_TRY(swimba_layer_fwd(&dc, (const char*)X_dev + r0 * xrow, w, init_c, (char*)y_dev + r0 * yrow, fin_c, nullptr,
                            nullptr, ws, ws_bytes, stream));
    SW_CUDA(cudaEventRecord(q->out[c], s));
    SW_CUDA(cudaStreamWaitEvent(q->d2h, q->out[c], 0));
    SW_CUDA(cudaMemcpy2DAsync((char*)y_host + h0 * yrow, hstride * yrow, (const char*)y_dev + r0 * yrow, len * yrow,
                              len * yrow, n, cudaMemcpyDeviceToHost, q->d2h));
  }
  SW_CUDA(cudaEventRecord(q->done, q->d2h));
  SW_CUDA(cudaStreamWaitEvent(s, q->done, 0));
  return SWIMBA_OK;
}

swimba_status swimba_step(const swimba_dims* dims, const void* X, const swimba_weights* w, float* state, void* y,
                          int32_t* topk_idx_out, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  if (d.T != 1) return SWIMBA_ERR_INVALID_ARG;
  SW_TRY(check_weights(w, true, true));
  if (!ok_ptr(X) || !ok_ptr(state) || !ok_ptr(y) || !ok_opt(topk_idx_out)) return SWIMBA_ERR_INVALID_ARG;
  SW_TRY(check_ws(d, ws, ws_bytes));
  WsPlan p = plan_workspace(d);
  char* b = (char*)ws;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t* idx = topk_idx_out ? topk_idx_out : (int32_t*)(b + p.topk_idx);
  float* wts = (float*)(b + p.topk_w);
  prof_begin(s);
  SW_TRY(run_front(d, X, w, b, p, idx, wts, 0, device_status(), s));
  const float *dt = (float*)(b + p.dt), *A = w->A;
  SW_TRY(run_mixed_a(d, w, idx, wts, b, p, &dt, &A, s));
  SW_CUDA(launch_step_update(d, b + p.bpi, b + p.xs, b + p.cpi, dt, A, state, y, s));
  prof_mark(s, "state_update");
  return SWIMBA_OK;
}

swimba_status swimba_separated_scan(const swimba_dims* dims, const void* B, const void* Xs, const void* Cpi,
                                    const float* dt, const float* A, const float* init_states, void* y,
                                    float* final_states, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  if (!ok_ptr(B) || !ok_ptr(Xs) || !ok_ptr(Cpi) || !ok_ptr(dt) || !A || !ok_ptr(y)) return SWIMBA_ERR_INVALID_ARG;
  if (!ok_opt(init_states) || !ok_opt(final_states)) return SWIMBA_ERR_INVALID_ARG;
  SW_TRY(check_ws(d, ws, ws_bytes));
  WsPlan p = plan_workspace(d);
  char* b = (char*)ws;
  const size_t one = (size_t)d.Bsz * d.H * d.N * d.P;
  prof_begin((cudaStream_t)stream);
  for (int j = 0; j < d.k; ++j) {
    ScanArgs a = mixed_scan_args(d, b, p, B, Xs, Cpi, dt, A, init_states ? init_states + j * one : nullptr, y,
                                 final_states ? final_states + j * one : nullptr, nullptr);
    a.key_slot0 = j; a.key_slots = 1; a.read_slot0 = j; a.read_slots = 1;
    a.accumulate_y = true; a.first_pass = j == 0; a.last_pass = j == d.k - 1;
    SW_TRY(run_scan(d, a, b, p, (cudaStream_t)stream));
  }
  prof_mark((cudaStream_t)stream, "separated_scan");
  return SWIMBA_OK;
}

swimba_status swimba_out_proj(const swimba_dims* dims, const void* y, const void* w_out, void* out, void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  if (!ok_ptr(y) || !ok_ptr(w_out) || !ok_ptr(out)) return SWIMBA_ERR_INVALID_ARG;
  unsigned* st = device_status();
  if (!st) return SWIMBA_ERR_CUDA;
  return cuda_status(launch_out_proj(d, y, w_out, out, st, (cudaStream_t)stream));
}

// Workspace of swimba_layer_bwd: the layer's own, then the gradient buffers (all fp32).
struct BwdPlan {
  size_t z, dbpi, dxs, dct, ddt, dpi, dg, du, dxp, poff, prow, rp_of_p, dzs, xsp, total;
};
static BwdPlan plan_bwd(const Dims& d) {
  BwdPlan q{};
  size_t o = align_up(plan_workspace(d).total, 256);
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  const size_t Mk = (size_t)d.M * d.k;
  q.z = take(Mk * d.We * 4);
  q.dbpi = take(Mk * d.GN * 4);
  q.dxs = take(Mk * d.HP * 4);
  q.dct = take((size_t)d.M * d.GN * 4);
  q.ddt = take((size_t)d.M * d.H * 4);
  q.dpi = take(Mk * 4);
  q.dg = take((size_t)d.M * d.E * 4);
  q.du = take((size_t)d.M * d.H * 4);
  q.dxp = take(Mk * d.D * 4);
  if (d.dtype == SWIMBA_BF16) {  // the tensor-core expert gradients' operands
    const size_t Rp = grad_tc_rows(d), Wp = (size_t)grad_tc_wp(d);
    q.poff = take((size_t)(d.E + 1) * 4);
    q.prow = take(Rp * 4);
    q.rp_of_p = take(Mk * 4);
    q.dzs = take(Rp * 2 * Wp * 2);
    q.xsp = take(Rp * d.D * 2);
  }
  q.total = o;
  return q;
}

size_t swimba_layer_bwd_workspace_size(const swimba_dims* dims) {
  Dims d;
  if (make_dims(dims, &d) != SWIMBA_OK) return 0;
  return plan_bwd(d).total;
}

swimba_status swimba_layer_bwd(const swimba_dims* dims, const void* X, const swimba_weights* w,
                               const float* init_state, const float* dy, float* dX, float* dW_router, float* dW_dt,
                               float* db_dt, float* dA, float* dW_exp, float* d_init, void* ws, size_t ws_bytes,
                               void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  SW_TRY(check_weights(w, true, true));
  if (w->A_exp || !w->A) return SWIMBA_ERR_UNSUPPORTED;
  if (!ok_ptr(X) || !ok_ptr(dy) || !ok_ptr(dX) || !ok_ptr(dW_router) || !ok_ptr(dW_dt) || !db_dt || !dA ||
      !ok_ptr(dW_exp) || !ok_opt(init_state) || !ok_opt(d_init))
    return SWIMBA_ERR_INVALID_ARG;
  if (scan_bwd_smem(d) > (size_t)227 * 1024) return SWIMBA_ERR_UNSUPPORTED;
  const BwdPlan q = plan_bwd(d);
  if (!ws || ((uintptr_t)ws & 15u) || ws_bytes < q.total) return SWIMBA_ERR_WORKSPACE;
  WsPlan p = plan_workspace(d);
  char* b = (char*)ws;
  cudaStream_t s = (cudaStream_t)stream;
  unsigned* st = device_status();
  if (!st) return SWIMBA_ERR_CUDA;
  int32_t* idx = (int32_t*)(b + p.topk_idx);
  float* wts = (float*)(b + p.topk_w);
  float* dt = (float*)(b + p.dt);
  prof_begin(s);
  // the forward's router, dispatch and mixed streams, and the raw projections z the mix's gradient reads:
  // one tensor-core GEMM writes both for bf16 layers; fp32 layers run the CUDA-core projection twice
  if (d.dtype == SWIMBA_BF16) {
    SW_TRY(run_front(d, X, w, b, p, idx, wts, 4, st, s, (float*)(b + q.z)));
  } else {
    SW_TRY(run_front(d, X, w, b, p, idx, wts, 0, st, s));
    SW_TRY(run_proj(d, X, w->w_exp, b, p, wts, 2, nullptr, nullptr, nullptr, (float*)(b + q.z), st, s));
  }
  SW_CUDA(launch_scan_bwd(d, b + p.bpi, b + p.xs, b + p.cpi, dt, w->A, init_state, dy, (float*)(b + q.dbpi),
                          (float*)(b + q.dxs), (float*)(b + q.dct), (float*)(b + q.ddt), dA, d_init,
                          (float*)(b + p.hstart), (float*)(b + p.schunk), (float*)(b + p.cslast), s));
  prof_mark(s, "ssd_scan_bwd");
  LayerBwdPtrs t{X, w->w_exp, w->w_router, w->w_dt, idx, wts, dt, (const float*)(b + q.ddt),
                 (const int32_t*)(b + p.perm), (const int32_t*)(b + p.tiles), (const int32_t*)(b + p.ntiles),
                 (const int32_t*)(b + p.offsets), (float*)(b + q.z), (const float*)(b + q.dbpi),
                 (const float*)(b + q.dxs), (const float*)(b + q.dct), (float*)(b + q.dpi), (float*)(b + q.dg),
                 (float*)(b + q.du), (float*)(b + q.dxp), dX, dW_router, dW_dt, db_dt, dW_exp,
                 b + p.xsorted, (int32_t*)(b + q.poff), (int32_t*)(b + q.prow), (int32_t*)(b + q.rp_of_p),
                 b + q.dzs, b + q.xsp, st};
  SW_CUDA(launch_layer_bwd_tail(d, t, 0, s));
  prof_mark(s, "mix_router_bwd");
  SW_CUDA(launch_layer_bwd_tail(d, t, 1, s));
  prof_mark(s, "expert_grad");
  SW_CUDA(launch_layer_bwd_tail(d, t, 2, s));
  prof_mark(s, "linear_bwd");
  return SWIMBA_OK;
}

swimba_status swimba_ssd_scan_bwd(const swimba_dims* dims, const void* Bpi, const void* Xs, const void* Cpi,
                                  const float* dt, const float* A, const float* init_state, const float* dy,
                                  float* dBpi, float* dXs, float* dCt, float* d_dt, float* dA, float* d_init,
                                  void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  SW_TRY(make_dims(dims, &d));
  if (!ok_ptr(Bpi) || !ok_ptr(Xs) || !ok_ptr(Cpi) || !ok_ptr(dt) || !A || !ok_ptr(dy) || !ok_ptr(dBpi) ||
      !ok_ptr(dXs) || !ok_ptr(dCt) || !ok_ptr(d_dt) || !dA || !ok_opt(init_state) || !ok_opt(d_init))
    return SWIMBA_ERR_INVALID_ARG;
  if (scan_bwd_smem(d) > (size_t)227 * 1024) return SWIMBA_ERR_UNSUPPORTED;
  SW_TRY(check_ws(d, ws, ws_bytes));
  WsPlan p = plan_workspace(d);
  char* b = (char*)ws;
  cudaStream_t s = (cudaStream_t)stream;
  prof_begin(s);
  SW_CUDA(launch_scan_bwd(d, Bpi, Xs, Cpi, dt, A, init_state, dy, dBpi, dXs, dCt, d_dt, dA, d_init,
                          (float*)(b + p.hstart), (float*)(b + p.schunk), (float*)(b + p.cslast), s));
  prof_mark(s, "ssd_scan_bwd");
  return SWIMBA_OK;
}

swimba_status swimba_check_device_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SWIMBA_ERR_CUDA;
  unsigned* st = device_status();
  if (!st) return SWIMBA_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, st, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SWIMBA_ERR_CUDA;
  if (v && cudaMemset(st, 0, sizeof(v)) != cudaSuccess) return SWIMBA_ERR_CUDA;
  if (v & ST_TIMEOUT) return SWIMBA_ERR_TIMEOUT;
  if (v & ST_RANGE) return SWIMBA_ERR_RANGE;
  if (v & ST_INDEX) return SWIMBA_ERR_INDEX;
  if (v & ST_UNSTABLE) return SWIMBA_ERR_UNSTABLE;
  return SWIMBA_OK;
}

swimba_status swimba_profile_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  if (enable && !g_prof.created) {
    for (int i = 0; i <= Profiler::kMax; ++i)
      if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) return SWIMBA_ERR_CUDA;
    g_prof.created = true;
  }
  g_prof.on = enable != 0;
  g_prof.n = 0;
  return SWIMBA_OK;
}

int swimba_profile_read(const char** names, float* ms, int max) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  if (!g_prof.created) return 0;
  const int n = g_prof.n < max ? g_prof.n : max;
  if (n > 0 && cudaEventSynchronize(g_prof.ev[n]) != cudaSuccess) return -1;
  for (int i = 0; i < n; ++i) {
    if (names) names[i] = g_prof.name[i];
    if (ms && cudaEventElapsedTime(&ms[i], g_prof.ev[i], g_prof.ev[i + 1]) != cudaSuccess) return -1;
  }
  return n;
}

long long swimba_launch_count(void) { return g_launches.load(); }

const char* swimba_status_string(swimba_status s) {
  switch (s) {
    case SWIMBA_OK: return "SWIMBA_OK";
    case SWIMBA_ERR_INVALID_ARG: return "SWIMBA_ERR_INVALID_ARG";
    case SWIMBA_ERR_UNSUPPORTED: return "SWIMBA_ERR_UNSUPPORTED";
    case SWIMBA_ERR_CUDA: return "SWIMBA_ERR_CUDA";
    case SWIMBA_ERR_WORKSPACE: return "SWIMBA_ERR_WORKSPACE";
    case SWIMBA_ERR_TIMEOUT: return "SWIMBA_ERR_TIMEOUT";
    case SWIMBA_ERR_RANGE: return "SWIMBA_ERR_RANGE";
    case SWIMBA_ERR_INDEX: return "SWIMBA_ERR_INDEX";
    case SWIMBA_ERR_UNSTABLE: return "SWIMBA_ERR_UNSTABLE";
  }
  return "SWIMBA_UNKNOWN_STATUS";
}

}  // extern "C"
