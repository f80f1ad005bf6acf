// Shared device/host helpers of libswimba (internal; not part of the C ABI).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "swimba.h"

namespace swimba {

// Bits of the device status word.
enum : unsigned { ST_TIMEOUT = 1u, ST_RANGE = 2u, ST_INDEX = 4u, ST_UNSTABLE = 8u };

// Largest finite fp16 value: mixed streams stored as fp16 must stay below it.
constexpr float kF16Max = 65504.f;

// Layer dimensions in the form the kernels use.
struct Dims {
  int Bsz, T, D, H, P, N, G, E, k, Q;
  int M;    // Bsz * T
  int HP;   // H * P
  int GN;   // G * N
  int We;   // HP + 2 * GN
  int nc;   // chunks per sequence
  int hpg;  // heads per group
  int dtype;
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }

template <class T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }

// True when v cannot be stored in T without overflow (fp16 only; fp32 streams take any value).
template <class T>
__device__ __forceinline__ bool out_of_range(float v) { return false; }
template <>
__device__ __forceinline__ bool out_of_range<__half>(float v) { return !(fabsf(v) <= kF16Max); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---------------------------------------------------------------------------------------------
// Workspace layout (every region 256-byte aligned).  The same plan serves every entry point.
struct WsPlan {
  size_t status;      // unsigned status word
  size_t topk_idx;    // int32 [M][k]
  size_t topk_w;      // f32 [M][k]
  size_t dt;          // f32 [M][H]
  size_t dA;          // f32 [M][H]  dt * A~ of the expert-mixed transition, and A = 1 [H] after it
  size_t ones;
  size_t dcounts;     // int32 [ndt][E]  per dispatch tile expert counts
  size_t dbase;       // int32 [ndt][E]  first sorted position of each (tile, expert)
  size_t offsets;     // int32 [E+1]
  size_t perm;        // int32 [M*k]
  size_t rowmeta;     // int2 [M*k]: per sorted row (pair index, router weight bits) for the GEMM epilogue
  size_t tiles;       // int32 [max_tiles][2]  GEMM row-tile schedule (expert, first sorted row)
  size_t ntiles;      // int32 [1]
  size_t xsorted;     // dtype [M*k][D] rows of X in sorted (expert-major) order
  size_t bpi, xs, cpi;  // stream dtype mixed streams
  size_t yintra;      // f32 [M][H][P]
  size_t ysum;        // f32 [M][H][P]  separated-scan accumulator
  size_t schunk;      // f32 [B][H][nc][N][P]  chunk-local end states
  size_t hstart;      // f32 [B][H][nc][N][P]  state before each chunk
  size_t cslast;      // f32 [B][H][nc]        total log-decay of each chunk
  size_t lb;          // unsigned: ticket counter (256 B) + [B*H][nsub] hand-off flags of the tensor-core scan
  size_t lb_bytes;
  size_t exch;        // f32 [B*H][nsub][N][P] state after each sub-chunk (tensor-core scan)
  size_t total;
};

constexpr int kDispatchTile = 1024;  // (token, slot) pairs per dispatch CTA
constexpr int kRowTile = 128;        // GEMM row tile of the schedule

inline int max_row_tiles(const Dims& d) { return ceil_div(d.M * d.k, kRowTile) + d.E; }
inline int dispatch_tiles(const Dims& d) { return ceil_div(d.M * d.k, kDispatchTile); }

size_t elem_bytes(int dtype);
int stream_dtype_of(int dtype);
WsPlan plan_workspace(const Dims& d);
// Validates the C ABI's dims and fills the kernels' form (every entry point's first step).
swimba_status make_dims(const swimba_dims* in, Dims* d);
// Device address of the current device's status word (looked up once per device; null on a CUDA error).
unsigned* device_status();

// ---------------------------------------------------------------------------------------------
// Kernel launchers (defined in the .cu files next to their kernels).  All return cudaError_t of the
// launch; `st` is the workspace status word.
// counts (nullable): [dispatch tile][E] table, zeroed by the caller, that the router increments for the
// (token, slot) pairs it routes (dispatch tile = pair index / kDispatchTile).
// after_zero: the stream's previous kernel is launch_zero_u32 clearing `counts` (and nothing else the router
// reads is produced by it): the tensor-core router then starts under programmatic dependent launch and waits
// for that kernel only before its first count.
cudaError_t launch_router(const Dims& d, const void* X, const swimba_weights& w, int32_t* idx, float* wts,
                          float* dt, int32_t* counts, unsigned* st, cudaStream_t s, bool after_zero = false);
// The tensor-core (tcgen05) router that launch_router prefers where it applies.
bool router_tc_supported(const Dims& d);
cudaError_t launch_router_tc(const Dims& d, const void* X, const swimba_weights& w, int32_t* idx, float* wts,
                             float* dt, int32_t* counts, unsigned* st, cudaStream_t s, bool after_zero);
// Zeroes n 32-bit words; lets the next kernel launch at once (it must wait before reading them).
cudaError_t launch_zero_u32(unsigned* p, size_t n, cudaStream_t s);
// rowmeta (nullable): per sorted row, (pair index p, router weight of p as float bits; 0 without topk_w).
// Pairs whose index lies outside [0, E) are left out of the sort and raise ST_INDEX in *st.
cudaError_t launch_dispatch(const Dims& d, const int32_t* idx, const WsPlan& p, char* ws, int32_t* offsets,
                            int32_t* perm, int2* rowmeta, const float* topk_w, unsigned* st, cudaStream_t s);
// bf16 layers: the same dispatch with the gather of X rows into expert-major order (xsorted) fused in.
cudaError_t launch_dispatch_gather(const Dims& d, const int32_t* idx, const int32_t* counts, const WsPlan& p, char* ws,
                                   int32_t* offsets, int32_t* perm, const float* topk_w, const void* X,
                                   cudaStream_t s);
// The layer's one-launch dispatch over counts the router produced (see launch_router).
cudaError_t launch_dispatch_fused(const Dims& d, const int32_t* idx, const int32_t* counts, const WsPlan& p, char* ws,
                                  int32_t* offsets, int32_t* perm, const float* topk_w, cudaStream_t s);
cudaError_t launch_gather_rows(const Dims& d, const void* X, const int32_t* perm, void* xsorted, cudaStream_t s);
// mode 0: fused mix (pi-scaled B and C), 1: fused mix with unscaled B, 2: raw Z (fp32)
cudaError_t launch_proj_simt(const Dims& d, const void* X, const void* w_exp, const int32_t* perm,
                             const int32_t* tiles, const int32_t* ntiles, const int32_t* offsets,
                             const float* topk_w, int mode, void* bpi, void* xs, void* cpi, float* Z, unsigned* st,
                             cudaStream_t s);
// Tensor-core version (bf16 X and weights, fp16 streams): A operand is xsorted (rows in expert order).
cudaError_t launch_proj_tc(const Dims& d, const void* xsorted, const void* w_exp, const int2* rowmeta,
                           const int32_t* tiles, const int32_t* ntiles, const int32_t* offsets, int mode, void* bpi,
                           void* xs, void* cpi, float* Z, unsigned* st, cudaStream_t s);
// Scan gradients (CUDA cores, 64-token sub-chunks): states of every sub-chunk in hstart/work, cs ends in cse.
int scan_bwd_subchunks(const Dims& d);
size_t scan_bwd_smem(const Dims& d);
cudaError_t launch_scan_bwd(const Dims& d, const void* bpi, const void* xs, const void* cpi, const float* dt,
                            const float* A, const float* init, const float* dy, float* dbpi, float* dxs, float* dct,
                            float* ddt, float* dA, float* dinit, float* hstart, float* work, float* cse,
                            cudaStream_t s);
// The layer gradients after the scan gradients (mix, router and dt, expert and router weight gradients, dX).
struct LayerBwdPtrs {
  const void* X; const void* w_exp; const void* w_r; const void* w_dt;
  const int32_t* idx; const float* wts; const float* dt; const float* ddt;
  const int32_t* perm; const int32_t* tiles; const int32_t* ntiles; const int32_t* offsets;
  float* z;      // [M*k][W_e] raw projections in, their gradients dz out
  const float* dbpi; const float* dxs; const float* dct;
  float* dpi; float* dg; float* du; float* dxp;
  float* dX; float* dW_r; float* dW_dt; float* db_dt; float* dW_exp;
  // bf16 layers: the tensor-core expert gradients' operands (gathered X rows, padded offsets, pair per
  // padded row and padded row per pair, dz split into bf16 hi/lo, padded X rows) and the device status word
  const void* xsorted; int32_t* poff; int32_t* prow; int32_t* rp_of_p; void* dzs; void* xsp; unsigned* st;
};
// The layer gradients after the scan's, in three parts: 0 mix and router, 1 expert products, 2 the router
// and dt weight gradients, db_dt and dX.
cudaError_t launch_layer_bwd_tail(const Dims& d, const LayerBwdPtrs& q, int part, cudaStream_t s);
// Rows of the padded sorted order (each expert's rows rounded up to 64) and W_e rounded up to 64.
size_t grad_tc_rows(const Dims& d);
int grad_tc_wp(const Dims& d);
cudaError_t launch_grad_tc_pack(const Dims& d, const void* xsorted, const int32_t* perm, const int32_t* offsets,
                                int32_t* poff, int32_t* prow, int32_t* rp_of_p, void* dzs, void* xsp, cudaStream_t s);
cudaError_t launch_grad_tc(const Dims& d, const void* w_exp, const int32_t* offsets, const int32_t* poff,
                           const int32_t* prow, const void* dzs, const void* xsp, float* dxp, float* dW_exp,
                           unsigned* st, cudaStream_t s);
cudaError_t launch_mixed_a(const Dims& d, const int32_t* idx, const float* wts, const float* A_exp, const float* dt,
                           float* dA, float* ones, unsigned* st, cudaStream_t s);
cudaError_t launch_out_proj(const Dims& d, const void* y, const void* w_out, void* out, unsigned* st,
                            cudaStream_t s);
cudaError_t launch_mix(const Dims& d, const float* Z, const float* topk_w, int flags, void* bpi, void* xs, void* cpi,
                       unsigned* st, cudaStream_t s);
// Chunked scan.  Slot ranges select which of the k per-token keys feed one trajectory and which
// readouts form C~: the mixed scan uses all k slots in one trajectory; the separated scan runs one
// slot per pass.
struct ScanArgs {
  const void* bpi; const void* xs; const void* cpi;  // streams, [M][k][...]
  const float* dt; const float* A;
  const float* init;  // [B][H][N][P] or null
  void* y;            // [M][H][P] out dtype
  bool accumulate_y;  // add into y (fp32 accumulator in yintra) instead of overwriting
  float* final_state; // or null
  float* hstart;      // [B][H][nc][N][P]
  float* chunk_states;  // [B][H][nc][N][P] caller's buffer or null (tensor-core scan writes it directly)
  float* schunk; float* cslast;
  float* yacc;        // [M][H][P] fp32: intra-chunk outputs
  float* ysum;        // [M][H][P] fp32: running sum over the separated design's trajectories
  int key_slot0;      // first slot used as a key
  int key_slots;      // number of key slots (k for the mixed scan, 1 for a separated trajectory)
  int read_slot0;     // first slot summed into the readout C~
  int read_slots;     // number of readout slots
  bool first_pass;    // separated scan: first slot initialises the fp32 accumulator
  bool last_pass;     // separated scan: last slot converts the accumulator to y
};
cudaError_t launch_scan_simt(const Dims& d, const ScanArgs& a, cudaStream_t s);
// Tensor-core scan (fp16 streams, N = 128, P in {64, 128}); `lb` must be zeroed before each launch.
bool scan_tc_supported(const Dims& d);
int scan_tc_subchunks(const Dims& d);
cudaError_t launch_scan_tc(const Dims& d, const ScanArgs& a, unsigned* lb, float* exch, unsigned* st,
                           cudaStream_t stream);
cudaError_t launch_step_update(const Dims& d, const void* bpi, const void* xs, const void* cpi, const float* dt,
                               const float* A, float* state, void* y, cudaStream_t s);
// Adds n to the library's launch counter (every launcher reports the kernels it issued).
void count_launches(int n);

// Programmatic dependent launch.  A kernel launched with launch_dependent() may be scheduled while the
// previous kernel in the stream is still finishing (once that kernel's CTAs have all signalled
// griddep_launch_dependents() or exited); it runs its prologue and calls griddep_wait() before it touches
// anything the previous kernels wrote.  Without the launch attribute griddep_wait() returns at once.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
// Raises a kernel's dynamic shared-memory limit on the current device to at least `bytes`; the driver is
// asked only when a larger limit than any earlier one is needed (the call costs microseconds of host time
// that would otherwise sit in front of every launch).
cudaError_t set_max_dynamic_smem(const void* kernel, size_t bytes);

}  // namespace swimba
