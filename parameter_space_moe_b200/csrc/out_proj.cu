// The layer's output projection out = y W_out^T (d_inner = H*P -> d_model).
//
// Paper: gist.science Technical Summary, Architecture Details -- the single shared recurrence's readout is
// followed by one output projection, shared by all experts (there is one recurrence, so there is one
// projection; no expert dimension).
//
// bf16 layers run it on the tensor cores (the dense schedule of the tcgen05 GEMM in proj_tc.cu, bf16 out).
// fp32 layers run the CUDA-core kernel below: their 1e-5 accuracy budget rules out tensor-core rounding.
// Each CTA computes a 128 x 64 tile with 256 threads (8 x 4 outputs per thread), K in steps of 16 staged
// through shared memory.
#include "common.cuh"

namespace swimba {

namespace {
constexpr int kOBM = 128, kOBN = 64, kOBK = 16;

__global__ void __launch_bounds__(256)
out_proj_simt_kernel(int M, int K, int N, const float* __restrict__ y, const float* __restrict__ W,
                     float* __restrict__ out) {
  __shared__ float As[kOBK][kOBM + 4];
  __shared__ float Bs[kOBK][kOBN + 4];
  const int m0 = blockIdx.x * kOBM, n0 = blockIdx.y * kOBN;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float acc[8][4] = {};
  for (int k0 = 0; k0 < K; k0 += kOBK) {
    for (int i = tid; i < kOBK * kOBM; i += 256) {
      const int r = i / kOBK, kk = i % kOBK;
      As[kk][r] = (m0 + r < M && k0 + kk < K) ? y[(size_t)(m0 + r) * K + k0 + kk] : 0.f;
    }
    for (int i = tid; i < kOBK * kOBN; i += 256) {
      const int c = i / kOBK, kk = i % kOBK;
      Bs[kk][c] = (n0 + c < N && k0 + kk < K) ? W[(size_t)(n0 + c) * K + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kOBK; ++kk) {
      float a[8], b[4];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = m0 + ty + 16 * i;
    if (r >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx + 16 * j;
      if (c < N) out[(size_t)r * N + c] = acc[i][j];
    }
  }
}
}  // namespace

cudaError_t launch_out_proj_tc(int M, int K, int N, const void* y, const void* w_out, void* out, unsigned* st,
                               cudaStream_t s);

cudaError_t launch_out_proj(const Dims& d, const void* y, const void* w_out, void* out, unsigned* st,
                            cudaStream_t s) {
  if (d.dtype == SWIMBA_BF16) return launch_out_proj_tc(d.M, d.HP, d.D, y, w_out, out, st, s);
  dim3 grid(ceil_div(d.M, kOBM), ceil_div(d.D, kOBN));
  out_proj_simt_kernel<<<grid, 256, 0, s>>>(d.M, d.HP, d.D, (const float*)y, (const float*)w_out, (float*)out);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swimba
