// Weight sharding: the split of W into the N shards of "Tensor Parallelism in
// Large Language Models" ("Column-Parallel Linear Layer": W = [W_1 ... W_N]
// along H_out; "Row-Parallel Linear Layer": W = [W_1; ...; W_N] along H_in;
// attention "Q, K, V Projections": W_Q, W_K, W_V sliced by whole heads),
// each shard stored transposed (K-major) as the GEMM kernels read it.
//
// A fourth kind packs the gate and up projections of a gated MLP (given as
// one [h][2F] matrix [W_gate | W_up]) so that each shard's columns alternate
// 128 gate features and the same 128 up features ("Partitioning the
// Multi-Layer Perceptron (MLP) Block": gate and up are both column-parallel).
//
// A fifth kind packs grouped-query QKV weights ("Grouped-Query Attention
// (GQA) Constraints"): shard i gets its n_q/N query heads and the key/value
// heads of their group(s) - n_kv/N of them, or one duplicated head when
// N > n_kv - as [Q_i | K_i | V_i].
//
// out[i][c][r] = W[row(i, r)][col(i, c)], an exact copy done as a 32 x 32
// shared-memory tiled transpose (coalesced reads along W's columns,
// coalesced writes along the shard's rows). One-time setup, HBM-bound.
#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

struct ShardMap {
  int64_t h_in, h_out;
  int64_t C, R;  // shard shape [C][R]
  int kind;      // 0 column, 1 row, 2 qkv heads, 3 gate/up interleaved, 4 GQA qkv
  int64_t hs;    // QKV: columns of one projection per shard (h / N); gate/up: F / N
  int64_t h3;    // QKV: h (columns of one projection); gate/up: F
  // GQA: query heads per shard, kv heads per shard, head dim, group size,
  // total query and kv heads
  int64_t qs, kvl, d, grp, nq, nkv;
};

constexpr int kGateUpBlock = 128;  // output features per gate (or up) block

__device__ __forceinline__ int64_t src_row(const ShardMap& m, int i, int64_t r) {
  return m.kind == 1 ? static_cast<int64_t>(i) * m.R + r : r;
}
__device__ __forceinline__ int64_t src_col(const ShardMap& m, int i, int64_t c) {
  if (m.kind == 0) return static_cast<int64_t>(i) * m.C + c;
  if (m.kind == 1) return c;
  if (m.kind == 3) {
    // block k of 2 x 128 shard columns: gate features k*128.., then up features
    const int64_t k = c / (2 * kGateUpBlock), w = c - k * 2 * kGateUpBlock;
    const int64_t f = static_cast<int64_t>(i) * m.hs + k * kGateUpBlock + (w % kGateUpBlock);
    return (w < kGateUpBlock) ? f : m.h3 + f;
  }
  if (m.kind == 4) {
    const int64_t qw = m.qs * m.d, kw = m.kvl * m.d;
    const int64_t first_kv = (static_cast<int64_t>(i) * m.qs) / m.grp;
    if (c < qw) return static_cast<int64_t>(i) * qw + c;
    if (c < qw + kw) return m.nq * m.d + first_kv * m.d + (c - qw);
    return (m.nq + m.nkv) * m.d + first_kv * m.d + (c - qw - kw);
  }
  const int64_t part = c / m.hs, within = c - part * m.hs;
  return part * m.h3 + static_cast<int64_t>(i) * m.hs + within;
}

__global__ void __launch_bounds__(256) shard_transpose_kernel(const uint16_t* __restrict__ W,
                                                              uint16_t* __restrict__ out,
                                                              ShardMap m) {
  __shared__ uint16_t tile[32][33];
  const int i = blockIdx.z;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int64_t c0 = static_cast<int64_t>(blockIdx.y) * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
#pragma unroll
  for (int k = 0; k < 32; k += 8) {
    const int64_t r = r0 + ty + k, c = c0 + tx;
    if (r < m.R && c < m.C) tile[ty + k][tx] = W[src_row(m, i, r) * m.h_out + src_col(m, i, c)];
  }
  __syncthreads();
  uint16_t* o = out + static_cast<int64_t>(i) * m.C * m.R;
#pragma unroll
  for (int k = 0; k < 32; k += 8) {
    const int64_t c = c0 + ty + k, r = r0 + tx;
    if (r < m.R && c < m.C) o[c * m.R + r] = tile[tx][ty + k];
  }
}

int launch_shard(const void* W, int64_t h_in, int64_t h_out, int n_shards, int kind,
                 int64_t head_dim, void* out, cudaStream_t s, int64_t n_q, int64_t n_kv) {
  ShardMap m;
  m.qs = m.kvl = m.d = m.grp = m.nq = m.nkv = 1;
  m.h_in = h_in;
  m.h_out = h_out;
  m.kind = kind;
  m.hs = 1;
  m.h3 = 1;
  if (kind == 0) {
    m.C = h_out / n_shards;
    m.R = h_in;
  } else if (kind == 1) {
    m.C = h_out;
    m.R = h_in / n_shards;
  } else if (kind == 2) {
    m.h3 = h_out / 3;
    m.hs = m.h3 / n_shards;
    m.C = 3 * m.hs;
    m.R = h_in;
  } else if (kind == 3) {
    m.h3 = h_out / 2;          // F
    m.hs = m.h3 / n_shards;    // F / N
    m.C = 2 * m.hs;
    m.R = h_in;
  } else {                     // GQA: h_out = (n_q + 2 n_kv) d
    m.nq = n_q;
    m.nkv = n_kv;
    m.d = head_dim;
    m.qs = n_q / n_shards;
    m.kvl = n_shards <= n_kv ? n_kv / n_shards : 1;
    m.grp = n_q / n_kv;
    m.C = (m.qs + 2 * m.kvl) * m.d;
    m.R = h_in;
  }
  const dim3 grid(static_cast<unsigned>((m.R + 31) / 32), static_cast<unsigned>((m.C + 31) / 32),
                  static_cast<unsigned>(n_shards));
  shard_transpose_kernel<<<grid, dim3(32, 8), 0, s>>>(static_cast<const uint16_t*>(W),
                                                      static_cast<uint16_t*>(out), m);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
