// swimba_dispatch_noalloc: expert dispatch for callers that cannot hand the library any scratch memory.
//
// Some callers cannot allocate device memory or pass a workspace: plugin-style hosts whose interface gives
// an operator only its inputs and outputs, and runtimes that plan all device memory once at start-up and
// refuse allocations afterwards.  This entry point serves them: the dispatch kernels' scratch (per-tile
// expert counts, per-tile bases, the grouped GEMM's row-tile schedule) lives in one fixed-size array
// compiled into the library, so the call allocates nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds kScratchBytes of
// it until the process exits.  In host code its name is only a host-side stand-in, so the device address
// is fetched with cudaGetSymbolAddress once per device (the first call on a device does it, with that
// device current) and handed to the kernels.  The address is kept for the life of the process, so a
// device reset (cudaDeviceReset) between calls is not supported.  All calls share the array and it keeps the last call's
// contents; every word the kernels read is written earlier in the same call, so nothing has to be
// cleared.  Two calls whose work overlaps on the GPU (different streams, or different host threads
// without ordering) race on the array.
#include <mutex>

#include "common.cuh"

namespace swimba {
namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;  // 1 MiB per device
static __device__ __align__(256) unsigned char g_dispatch_scratch[kScratchBytes];

// Device address of g_dispatch_scratch on the current device (looked up once per device).
cudaError_t scratch_address(char** out) {
  static std::mutex mu;
  static char* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<char*>(p);
  }
  *out = addr[dev];
  return cudaSuccess;
}

// The regions launch_dispatch uses, laid out inside the fixed array instead of a caller workspace.
bool scratch_plan(const Dims& d, WsPlan* p) {
  WsPlan q{};
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
  q.dcounts = take((size_t)dispatch_tiles(d) * d.E * 4);
  q.dbase = take((size_t)dispatch_tiles(d) * d.E * 4);
  q.tiles = take((size_t)max_row_tiles(d) * 8);
  q.ntiles = take(4);
  q.total = o;
  *p = q;
  return o <= kScratchBytes;
}

}  // namespace
}  // namespace swimba

using namespace swimba;

extern "C" swimba_status swimba_dispatch_noalloc(const swimba_dims* dims, const int32_t* topk_idx,
                                                 int32_t* expert_offsets, int32_t* perm, void* stream) {
  // the same dims rules and status codes as swimba_dispatch
  Dims d{};
  const swimba_status ds = make_dims(dims, &d);
  if (ds != SWIMBA_OK) return ds;
  if (!topk_idx || !expert_offsets || !perm) return SWIMBA_ERR_INVALID_ARG;
  if (((uintptr_t)topk_idx | (uintptr_t)expert_offsets | (uintptr_t)perm) & 15u) return SWIMBA_ERR_INVALID_ARG;
  WsPlan p;
  if (!scratch_plan(d, &p)) return SWIMBA_ERR_WORKSPACE;  // needs more than the fixed 1 MiB scratch
  char* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return SWIMBA_ERR_CUDA;
  unsigned* st = device_status();
  if (!st) return SWIMBA_ERR_CUDA;
  return launch_dispatch(d, topk_idx, p, scratch, expert_offsets, perm, nullptr, nullptr, st,
                         (cudaStream_t)stream) == cudaSuccess
             ? SWIMBA_OK
             : SWIMBA_ERR_CUDA;
}
