// Element-wise and column-reduction kernels of the MLP backward pass.
//
// "Tensor Parallelism in Large Language Models", MLP block: the backward of
// the paired column -> row layers needs exactly one all-reduce, of the input
// gradient across the column-parallel layer. The GEMMs of that backward run
// in gemm_tcgen05.cu; here are the HBM-bound pieces around them: H = GeLU(Z)
// from the recomputed pre-activation (for dB), and the bias gradients as
// column sums over the token rows (two deterministic passes: per-slab
// partial sums, then their sum in slab order).
#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

__global__ void __launch_bounds__(256) gelu_bf16_kernel(const uint16_t* __restrict__ Z,
                                                        uint16_t* __restrict__ H, int64_t n8) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 z = __ldg(reinterpret_cast<const uint4*>(Z) + i);
    uint4 o;
    o.x = pack_bf16x2(gelu_erf(bf16_lo(z.x)), gelu_erf(bf16_hi(z.x)));
    o.y = pack_bf16x2(gelu_erf(bf16_lo(z.y)), gelu_erf(bf16_hi(z.y)));
    o.z = pack_bf16x2(gelu_erf(bf16_lo(z.z)), gelu_erf(bf16_hi(z.z)));
    o.w = pack_bf16x2(gelu_erf(bf16_lo(z.w)), gelu_erf(bf16_hi(z.w)));
    reinterpret_cast<uint4*>(H)[i] = o;
  }
}

// partial[g][s][c] = sum over rows r in slab s of X[g][r][c] (8 columns per thread)
__global__ void __launch_bounds__(128) colsum_partial_kernel(const uint16_t* __restrict__ X,
                                                             float* __restrict__ partial,
                                                             int rows, int cols, int slabs) {
  const int c8 = blockIdx.x * blockDim.x + threadIdx.x;
  const int s = blockIdx.y, g = blockIdx.z;
  if (c8 * 8 >= cols) return;
  const int r0 = static_cast<int>((static_cast<int64_t>(rows) * s) / slabs);
  const int r1 = static_cast<int>((static_cast<int64_t>(rows) * (s + 1)) / slabs);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const uint16_t* base = X + static_cast<int64_t>(g) * rows * cols + c8 * 8;
  for (int r = r0; r < r1; ++r) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(r) * cols));
    acc[0] += bf16_lo(v.x); acc[1] += bf16_hi(v.x);
    acc[2] += bf16_lo(v.y); acc[3] += bf16_hi(v.y);
    acc[4] += bf16_lo(v.z); acc[5] += bf16_hi(v.z);
    acc[6] += bf16_lo(v.w); acc[7] += bf16_hi(v.w);
  }
  float* out = partial + (static_cast<int64_t>(g) * slabs + s) * cols + c8 * 8;
#pragma unroll
  for (int e = 0; e < 8; ++e) out[e] = acc[e];
}

__global__ void __launch_bounds__(256) colsum_final_kernel(const float* __restrict__ partial,
                                                           float* __restrict__ out, int cols,
                                                           int slabs, int groups) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i >= static_cast<int64_t>(groups) * cols) return;
  const int64_t g = i / cols, c = i - g * cols;
  float t = 0.f;
  for (int s = 0; s < slabs; ++s) t += partial[(g * slabs + s) * cols + c];
  out[i] = t;
}

int launch_gelu_bf16(const void* Z, void* H, int64_t n, cudaStream_t s, int num_sms) {
  const int64_t n8 = n / 8;
  int64_t blocks = (n8 + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  gelu_bf16_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint16_t*>(Z),
                                          static_cast<uint16_t*>(H), n8);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

int launch_colsum(const void* X, int groups, int rows, int cols, float* partial, int slabs,
                  float* out, cudaStream_t s) {
  const dim3 grid((cols / 8 + 127) / 128, slabs, groups);
  colsum_partial_kernel<<<grid, 128, 0, s>>>(static_cast<const uint16_t*>(X), partial, rows, cols,
                                             slabs);
  const int64_t n = static_cast<int64_t>(groups) * cols;
  colsum_final_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(partial, out, cols,
                                                                             slabs, groups);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
