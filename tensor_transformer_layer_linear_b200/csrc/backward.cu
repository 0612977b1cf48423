// Column reductions of the backward passes: the bias gradients.
//
// "Tensor Parallelism in Large Language Models", MLP block: the backward of
// the paired column -> row layers needs exactly one all-reduce, of the input
// gradient across the column-parallel layer. The GEMMs of that backward run
// in gemm_tcgen05.cu; the bias gradients are column sums of the output
// gradients over the token rows, done here in two deterministic passes
// (per-slab partial sums, then their sum in slab order).
#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

constexpr int kColsumThreads = 128;
constexpr int kColsumUnroll = 16;  // rows whose loads are in flight together
constexpr int kColsumRows = 32;    // target rows per slab

// partial[g][s][c] = sum over rows r in slab s of X[g][r][c] (8 columns per
// thread, rows added in increasing order)
__global__ void __launch_bounds__(kColsumThreads) colsum_partial_kernel(
    const uint16_t* __restrict__ X, float* __restrict__ partial, int rows, int cols, int slabs) {
  const int c8 = blockIdx.x * blockDim.x + threadIdx.x;
  const int s = blockIdx.y, g = blockIdx.z;
  if (c8 * 8 >= cols) return;
  const int r0 = static_cast<int>((static_cast<int64_t>(rows) * s) / slabs);
  const int r1 = static_cast<int>((static_cast<int64_t>(rows) * (s + 1)) / slabs);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const uint16_t* base = X + static_cast<int64_t>(g) * rows * cols + c8 * 8;
  auto add = [&](const uint4& v) {
    acc[0] += bf16_lo(v.x); acc[1] += bf16_hi(v.x);
    acc[2] += bf16_lo(v.y); acc[3] += bf16_hi(v.y);
    acc[4] += bf16_lo(v.z); acc[5] += bf16_hi(v.z);
    acc[6] += bf16_lo(v.w); acc[7] += bf16_hi(v.w);
  };
  int r = r0;
  for (; r + kColsumUnroll <= r1; r += kColsumUnroll) {
    uint4 v[kColsumUnroll];
#pragma unroll
    for (int u = 0; u < kColsumUnroll; ++u)
      v[u] = __ldg(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(r + u) * cols));
#pragma unroll
    for (int u = 0; u < kColsumUnroll; ++u) add(v[u]);
  }
  for (; r < r1; ++r)
    add(__ldg(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(r) * cols)));
  float4* out = reinterpret_cast<float4*>(partial + (static_cast<int64_t>(g) * slabs + s) * cols +
                                          c8 * 8);
  out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// out[g][c] = sum over slabs of partial[g][s][c]: 32 columns per CTA, eight
// threads per column each summing every eighth slab, then those eight sums in
// a fixed order.
__global__ void __launch_bounds__(256) colsum_final_kernel(const float* __restrict__ partial,
                                                           float* __restrict__ out, int cols,
                                                           int slabs, int groups) {
  __shared__ float part[8][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t i = blockIdx.x * 32LL + tx;
  const bool live = i < static_cast<int64_t>(groups) * cols;
  float t = 0.f;
  if (live) {
    const int64_t g = i / cols, c = i - g * cols;
    const float* col = partial + g * slabs * cols + c;
    int s = ty;
    for (; s + 8 * 7 < slabs; s += 8 * 8) {  // eight loads in flight, added in slab order
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = col[static_cast<int64_t>(s + 8 * u) * cols];
#pragma unroll
      for (int u = 0; u < 8; ++u) t += v[u];
    }
    for (; s < slabs; s += 8) t += col[static_cast<int64_t>(s) * cols];
  }
  part[ty][tx] = t;
  __syncthreads();
  if (ty == 0 && live) {
    float r = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) r += part[k][tx];
    out[i] = r;
  }
}

int launch_colsum(const void* X, int groups, int rows, int cols, float* partial, int max_slabs,
                  float* out, cudaStream_t s, int num_sms) {
  const int col_blocks = (cols / 8 + kColsumThreads - 1) / kColsumThreads;
  // about kColsumRows rows per slab, at least 8 CTAs per SM when rows allow
  int slabs = (rows + kColsumRows - 1) / kColsumRows;
  const int fill = (8 * num_sms + col_blocks * groups - 1) / (col_blocks * groups);
  if (slabs < fill) slabs = fill < rows / 8 ? fill : rows / 8;
  if (slabs > max_slabs) slabs = max_slabs;
  if (slabs < 1) slabs = 1;
  const dim3 grid(col_blocks, slabs, groups);
  colsum_partial_kernel<<<grid, kColsumThreads, 0, s>>>(static_cast<const uint16_t*>(X), partial,
                                                        rows, cols, slabs);
  const int64_t n = static_cast<int64_t>(groups) * cols;
  colsum_final_kernel<<<static_cast<unsigned>((n + 31) / 32), 256, 0, s>>>(partial, out, cols,
                                                                           slabs, groups);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

int launch_slab_sum(const float* partial, int slabs, int cols, float* out, cudaStream_t s) {
  colsum_final_kernel<<<static_cast<unsigned>((cols + 31) / 32), 256, 0, s>>>(partial, out, cols,
                                                                              slabs, 1);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
