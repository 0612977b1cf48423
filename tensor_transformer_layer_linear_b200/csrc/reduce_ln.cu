// The block-output reduction of the N row-parallel partials, and the
// replicated LayerNorm around the blocks.
//
// "Tensor Parallelism in Large Language Models", "Row-Parallel Linear
// Layer": the true output is Y = sum_i Y_i, obtained across GPUs by an
// all-reduce sum. With the N shards held as N buffers of one GPU the
// all-reduce is a streaming sum of N fp32 partials, fused here with the
// output bias and the residual add (each added once), one bf16 rounding.
// The kernel is HBM-bound: it reads N*rows*h*4 + rows*h*2 + h*2 bytes and
// writes rows*h*2, with 128-bit loads and stores, partials streamed with
// evict-first loads, grid sized to a multiple of the SM count.
//
// LayerNorm ("Sequence Parallelism": LayerNorm, dropout and residual adds are
// replicated on every rank): one CTA per token row, fp32 statistics with
// warp shuffles, population variance; it can be fused behind the sum so the
// residual stream h1 and LN(h1) leave in one pass.
#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

__device__ __forceinline__ void add_bf16x8(float (&a)[8], const uint4& b) {
  a[0] += bf16_lo(b.x); a[1] += bf16_hi(b.x);
  a[2] += bf16_lo(b.y); a[3] += bf16_hi(b.y);
  a[4] += bf16_lo(b.z); a[5] += bf16_hi(b.z);
  a[6] += bf16_lo(b.w); a[7] += bf16_hi(b.w);
}

__device__ __forceinline__ uint4 to_bf16x8(const float (&a)[8]) {
  uint4 o;
  o.x = pack_bf16x2(a[0], a[1]);
  o.y = pack_bf16x2(a[2], a[3]);
  o.z = pack_bf16x2(a[4], a[5]);
  o.w = pack_bf16x2(a[6], a[7]);
  return o;
}

// Sum of the N partials at element offset e (8 consecutive fp32), in shard
// order 0..N-1. NS > 0: compile-time N (all loads issued before the adds).
template <int NS>
__device__ __forceinline__ void sum_partials8(const float* __restrict__ P, int n_shards,
                                              int64_t stride, int64_t e, float (&acc)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  if constexpr (NS > 0) {
    float4 v[NS][2];
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      const float4* src = reinterpret_cast<const float4*>(P + s * stride + e);
      v[s][0] = __ldcs(src);
      v[s][1] = __ldcs(src + 1);
    }
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      acc[0] += v[s][0].x; acc[1] += v[s][0].y; acc[2] += v[s][0].z; acc[3] += v[s][0].w;
      acc[4] += v[s][1].x; acc[5] += v[s][1].y; acc[6] += v[s][1].z; acc[7] += v[s][1].w;
    }
  } else {
    for (int s = 0; s < n_shards; ++s) {
      const float4* src = reinterpret_cast<const float4*>(P + s * stride + e);
      const float4 a = __ldcs(src), b = __ldcs(src + 1);
      acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
      acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    }
  }
}

// Y = sum_i P_i + bias + residual. With sp.n > 0 the residual is read from,
// and Y written to, the sequence-sharded layout (the reduce-scatter).
template <int NS>
__global__ void __launch_bounds__(256) reduce_partials_kernel(
    const float* __restrict__ P, int n_shards, int64_t n_elems, int h,
    const uint16_t* __restrict__ bias, const uint16_t* __restrict__ res,
    uint16_t* __restrict__ Y, SeqShard sp) {
  const int64_t n8 = n_elems >> 3;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = i << 3;
    float acc[8];
    sum_partials8<NS>(P, n_shards, n_elems, e, acc);
    const int64_t m = e / h;
    const int64_t col = e - m * h;
    const int64_t d = seq_shard_row(sp, m) * h + col;
    if (bias != nullptr) add_bf16x8(acc, __ldg(reinterpret_cast<const uint4*>(bias + col)));
    if (res != nullptr) add_bf16x8(acc, __ldg(reinterpret_cast<const uint4*>(res + d)));
    *reinterpret_cast<uint4*>(Y + d) = to_bf16x8(acc);
  }
}

// X[b S + s] = X_shards[s / (S/N)][b][s % (S/N)]: the all-gather along the
// sequence before a column-parallel layer (16-byte copies).
__global__ void __launch_bounds__(256) all_gather_sequence_kernel(
    const uint16_t* __restrict__ Xs, uint16_t* __restrict__ X, int64_t n_elems, int h,
    SeqShard sp) {
  const int64_t n8 = n_elems >> 3;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = i << 3;
    const int64_t m = e / h;
    const int64_t col = e - m * h;
    *reinterpret_cast<uint4*>(X + e) =
        __ldcs(reinterpret_cast<const uint4*>(Xs + seq_shard_row(sp, m) * h + col));
  }
}

template <int THREADS>
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < THREADS / 32; ++i) t += red[i];
  __syncthreads();
  return t;
}

// One CTA of kRowThreads threads per row; CH = 8-element chunks per thread
// (h <= CH * 8 * kRowThreads). The plain LayerNorm (no partials) uses 128
// threads per row so that more rows, and more loads, are in flight per SM.
// With sp.n > 0 the residual is read from and Y_sum written to the
// sequence-sharded layout, and Y_ln is written in token order when ln_natural
// (the sharded LayerNorm followed by the all-gather) or sharded otherwise.
template <int CH, int NS, int kRowThreads>
__global__ void __launch_bounds__(kRowThreads) rows_sum_ln_kernel(
    const float* __restrict__ P, int n_shards, int64_t stride, int h,
    const uint16_t* __restrict__ bias, const uint16_t* __restrict__ res,
    const uint16_t* __restrict__ gamma, const uint16_t* __restrict__ beta, float eps,
    uint16_t* __restrict__ Ysum, uint16_t* __restrict__ Yln, SeqShard sp, int ln_natural) {
  __shared__ float red[kRowThreads / 32];
  const int64_t row_off = static_cast<int64_t>(blockIdx.x) * h;
  const int64_t sh_off = seq_shard_row(sp, blockIdx.x) * h;  // same row, sharded layout
  const int64_t ln_off = ln_natural ? row_off : sh_off;
  const int nch = h >> 3;
  float v[CH][8];
  float s = 0.f;
  // gamma and beta of this thread's chunks, in flight with the row's loads
  // (not one L2 round trip per chunk after the statistics); wide rows load
  // them per chunk instead, to stay within the register budget
  constexpr bool kPre = CH <= 4;
  uint4 gq[kPre ? CH : 1], bq[kPre ? CH : 1];
#pragma unroll
  for (int c = 0; c < (kPre ? CH : 0); ++c) {
    const int ch = threadIdx.x + c * kRowThreads;
    gq[c] = bq[c] = make_uint4(0u, 0u, 0u, 0u);
    if (Yln != nullptr && ch < nch) {
      gq[c] = __ldg(reinterpret_cast<const uint4*>(gamma + (ch << 3)));
      bq[c] = __ldg(reinterpret_cast<const uint4*>(beta + (ch << 3)));
    }
  }
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int ch = threadIdx.x + c * kRowThreads;
    if (ch < nch) {
      const int64_t e = row_off + (ch << 3);
      if (n_shards > 0) {
        sum_partials8<NS>(P, n_shards, stride, e, v[c]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[c][j] = 0.f;
      }
      const int64_t es = sh_off + (ch << 3);
      if (bias != nullptr) add_bf16x8(v[c], __ldg(reinterpret_cast<const uint4*>(bias + (ch << 3))));
      if (res != nullptr) add_bf16x8(v[c], __ldg(reinterpret_cast<const uint4*>(res + es)));
      const uint4 o = to_bf16x8(v[c]);
      if (Ysum != nullptr) *reinterpret_cast<uint4*>(Ysum + es) = o;
      // statistics of the rounded values, as a separate LayerNorm would see them
      v[c][0] = bf16_lo(o.x); v[c][1] = bf16_hi(o.x);
      v[c][2] = bf16_lo(o.y); v[c][3] = bf16_hi(o.y);
      v[c][4] = bf16_lo(o.z); v[c][5] = bf16_hi(o.z);
      v[c][6] = bf16_lo(o.w); v[c][7] = bf16_hi(o.w);
#pragma unroll
      for (int j = 0; j < 8; ++j) s += v[c][j];
    }
  }
  if (Yln == nullptr) return;
  const float mean = block_sum<kRowThreads>(s, red) / static_cast<float>(h);
  float q = 0.f;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int ch = threadIdx.x + c * kRowThreads;
    if (ch < nch) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float d = v[c][j] - mean;
        q += d * d;
      }
    }
  }
  const float var = block_sum<kRowThreads>(q, red) / static_cast<float>(h);
  const float rstd = rsqrtf(var + eps);
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int ch = threadIdx.x + c * kRowThreads;
    if (ch < nch) {
      const uint4 g = kPre ? gq[kPre ? c : 0] : __ldg(reinterpret_cast<const uint4*>(gamma + (ch << 3)));
      const uint4 b = kPre ? bq[kPre ? c : 0] : __ldg(reinterpret_cast<const uint4*>(beta + (ch << 3)));
      float gv[8] = {bf16_lo(g.x), bf16_hi(g.x), bf16_lo(g.y), bf16_hi(g.y),
                     bf16_lo(g.z), bf16_hi(g.z), bf16_lo(g.w), bf16_hi(g.w)};
      float bv[8] = {bf16_lo(b.x), bf16_hi(b.x), bf16_lo(b.y), bf16_hi(b.y),
                     bf16_lo(b.z), bf16_hi(b.z), bf16_lo(b.w), bf16_hi(b.w)};
      float y[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) y[j] = (v[c][j] - mean) * rstd * gv[j] + bv[j];
      *reinterpret_cast<uint4*>(Yln + ln_off + (ch << 3)) = to_bf16x8(y);
    }
  }
}

// The plain LayerNorm (no partials to sum): one warp per token row, eight
// rows per CTA, every 16-byte load of the row issued before the first
// reduction and warp shuffles only, so that a whole wave of rows streams at
// once. CHW = 8-element chunks per lane (h <= CHW * 256); lane l holds chunks
// l, l + 32, ... so each step of the warp reads 512 contiguous bytes. The
// row value is bias + residual rounded to bf16 (written to Y_sum when given);
// statistics are taken over the rounded values, population variance. gamma
// and beta are staged in shared memory once per CTA (read per chunk from
// global memory they cost one L2 round trip per chunk after the statistics).
template <int CHW>
__global__ void __launch_bounds__(256) layernorm_rows_warp_kernel(
    int64_t rows, int h, const uint16_t* __restrict__ bias, const uint16_t* __restrict__ res,
    const uint16_t* __restrict__ gamma, const uint16_t* __restrict__ beta, float eps,
    uint16_t* __restrict__ Ysum, uint16_t* __restrict__ Yln, SeqShard sp, int ln_natural) {
  extern __shared__ uint4 gb_s[];  // [2][h / 8]: gamma, then beta
  const int lane = threadIdx.x & 31;
  const int nch = h >> 3;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const bool active = row < rows;
  const int64_t row_off = row * h;
  const int64_t sh_off = active ? seq_shard_row(sp, row) * h : 0;  // same row, sharded layout
  const int64_t ln_off = ln_natural ? row_off : sh_off;
  // the row's loads go out first; gamma and beta are staged while they fly
  uint4 x[CHW];
#pragma unroll
  for (int c = 0; c < CHW; ++c) {
    const int ch = lane + 32 * c;
    x[c] = make_uint4(0u, 0u, 0u, 0u);
    if (active && res != nullptr && ch < nch)
      x[c] = __ldg(reinterpret_cast<const uint4*>(res + sh_off + (ch << 3)));
  }
  if (Yln != nullptr) {
    for (int i = threadIdx.x; i < nch; i += blockDim.x) {
      gb_s[i] = __ldg(reinterpret_cast<const uint4*>(gamma) + i);
      gb_s[nch + i] = __ldg(reinterpret_cast<const uint4*>(beta) + i);
    }
  }
  __syncthreads();
  if (!active) return;
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < CHW; ++c) {
    const int ch = lane + 32 * c;
    if (ch < nch) {
      float v[8] = {bf16_lo(x[c].x), bf16_hi(x[c].x), bf16_lo(x[c].y), bf16_hi(x[c].y),
                    bf16_lo(x[c].z), bf16_hi(x[c].z), bf16_lo(x[c].w), bf16_hi(x[c].w)};
      if (bias != nullptr) {
        add_bf16x8(v, __ldg(reinterpret_cast<const uint4*>(bias + (ch << 3))));
        x[c] = to_bf16x8(v);
        v[0] = bf16_lo(x[c].x); v[1] = bf16_hi(x[c].x);
        v[2] = bf16_lo(x[c].y); v[3] = bf16_hi(x[c].y);
        v[4] = bf16_lo(x[c].z); v[5] = bf16_hi(x[c].z);
        v[6] = bf16_lo(x[c].w); v[7] = bf16_hi(x[c].w);
      }
      if (Ysum != nullptr) *reinterpret_cast<uint4*>(Ysum + sh_off + (ch << 3)) = x[c];
#pragma unroll
      for (int j = 0; j < 8; ++j) s += v[j];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / static_cast<float>(h);
  float q = 0.f;
#pragma unroll
  for (int c = 0; c < CHW; ++c) {
    const int ch = lane + 32 * c;
    if (ch < nch) {
      const float v[8] = {bf16_lo(x[c].x), bf16_hi(x[c].x), bf16_lo(x[c].y), bf16_hi(x[c].y),
                          bf16_lo(x[c].z), bf16_hi(x[c].z), bf16_lo(x[c].w), bf16_hi(x[c].w)};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float d = v[j] - mean;
        q += d * d;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = rsqrtf(q / static_cast<float>(h) + eps);
  if (Yln == nullptr) return;
#pragma unroll
  for (int c = 0; c < CHW; ++c) {
    const int ch = lane + 32 * c;
    if (ch < nch) {
      const uint4 g = gb_s[ch];
      const uint4 b = gb_s[nch + ch];
      const float v[8] = {bf16_lo(x[c].x), bf16_hi(x[c].x), bf16_lo(x[c].y), bf16_hi(x[c].y),
                          bf16_lo(x[c].z), bf16_hi(x[c].z), bf16_lo(x[c].w), bf16_hi(x[c].w)};
      const float gv[8] = {bf16_lo(g.x), bf16_hi(g.x), bf16_lo(g.y), bf16_hi(g.y),
                           bf16_lo(g.z), bf16_hi(g.z), bf16_lo(g.w), bf16_hi(g.w)};
      const float bv[8] = {bf16_lo(b.x), bf16_hi(b.x), bf16_lo(b.y), bf16_hi(b.y),
                           bf16_lo(b.z), bf16_hi(b.z), bf16_lo(b.w), bf16_hi(b.w)};
      float y[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) y[j] = (v[j] - mean) * rstd * gv[j] + bv[j];
      *reinterpret_cast<uint4*>(Yln + ln_off + (ch << 3)) = to_bf16x8(y);
    }
  }
}

template <int CHW>
static void launch_ln_warp(int64_t rows, int64_t h, const void* bias, const void* residual,
                           const void* gamma, const void* beta, float eps, void* Y_sum,
                           void* Y_ln, cudaStream_t s, SeqShard sp, int ln_nat) {
  const dim3 grid(static_cast<unsigned>((rows + 7) / 8));
  const size_t smem = Y_ln != nullptr ? static_cast<size_t>(h / 8) * 2 * sizeof(uint4) : 0;
  layernorm_rows_warp_kernel<CHW><<<grid, 256, smem, s>>>(
      rows, static_cast<int>(h), static_cast<const uint16_t*>(bias),
      static_cast<const uint16_t*>(residual), static_cast<const uint16_t*>(gamma),
      static_cast<const uint16_t*>(beta), eps, static_cast<uint16_t*>(Y_sum),
      static_cast<uint16_t*>(Y_ln), sp, ln_nat);
}

int launch_reduce(const float* P, int n_shards, int64_t rows, int64_t h, const void* bias,
                  const void* residual, void* Y, cudaStream_t s, int num_sms, int sp_n,
                  int sp_batch, int sp_seq) {
  const SeqShard sp{sp_n, sp_batch, sp_seq};
  const int64_t n = rows * h;
  const int64_t n8 = n / 8;
  int64_t blocks = (n8 + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  auto b = static_cast<const uint16_t*>(bias);
  auto r = static_cast<const uint16_t*>(residual);
  auto y = static_cast<uint16_t*>(Y);
  const int hh = static_cast<int>(h);
  switch (n_shards) {
    case 1: reduce_partials_kernel<1><<<blocks, 256, 0, s>>>(P, 1, n, hh, b, r, y, sp); break;
    case 2: reduce_partials_kernel<2><<<blocks, 256, 0, s>>>(P, 2, n, hh, b, r, y, sp); break;
    case 4: reduce_partials_kernel<4><<<blocks, 256, 0, s>>>(P, 4, n, hh, b, r, y, sp); break;
    case 8: reduce_partials_kernel<8><<<blocks, 256, 0, s>>>(P, 8, n, hh, b, r, y, sp); break;
    case 16: reduce_partials_kernel<16><<<blocks, 256, 0, s>>>(P, 16, n, hh, b, r, y, sp); break;
    default: reduce_partials_kernel<0><<<blocks, 256, 0, s>>>(P, n_shards, n, hh, b, r, y, sp); break;
  }
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

template <int CH, int THREADS>
static void launch_rows_ch(const float* P, int n_shards, int64_t rows, int64_t h, const void* bias,
                           const void* residual, const void* gamma, const void* beta, float eps,
                           void* Y_sum, void* Y_ln, cudaStream_t s, SeqShard sp, int ln_nat) {
  auto b = static_cast<const uint16_t*>(bias);
  auto r = static_cast<const uint16_t*>(residual);
  auto g = static_cast<const uint16_t*>(gamma);
  auto be = static_cast<const uint16_t*>(beta);
  auto ys = static_cast<uint16_t*>(Y_sum);
  auto yl = static_cast<uint16_t*>(Y_ln);
  const int64_t stride = rows * h;
  const int hh = static_cast<int>(h);
  const dim3 grid(static_cast<unsigned>(rows));
  switch (n_shards) {
    case 4: rows_sum_ln_kernel<CH, 4, THREADS><<<grid, THREADS, 0, s>>>(P, 4, stride, hh, b, r, g, be, eps, ys, yl, sp, ln_nat); break;
    case 8: rows_sum_ln_kernel<CH, 8, THREADS><<<grid, THREADS, 0, s>>>(P, 8, stride, hh, b, r, g, be, eps, ys, yl, sp, ln_nat); break;
    default: rows_sum_ln_kernel<CH, 0, THREADS><<<grid, THREADS, 0, s>>>(P, n_shards, stride, hh, b, r, g, be, eps, ys, yl, sp, ln_nat); break;
  }
}

template <int THREADS>
static void launch_rows(const float* P, int n_shards, int64_t rows, int64_t h, const void* bias,
                        const void* residual, const void* gamma, const void* beta, float eps,
                        void* Y_sum, void* Y_ln, cudaStream_t s, SeqShard sp, int ln_nat) {
  const int64_t nch = h / 8;
  if (nch <= THREADS) launch_rows_ch<1, THREADS>(P, n_shards, rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp, ln_nat);
  else if (nch <= 2 * THREADS) launch_rows_ch<2, THREADS>(P, n_shards, rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp, ln_nat);
  else if (nch <= 4 * THREADS) launch_rows_ch<4, THREADS>(P, n_shards, rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp, ln_nat);
  else if (nch <= 8 * THREADS) launch_rows_ch<8, THREADS>(P, n_shards, rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp, ln_nat);
  else launch_rows_ch<16, THREADS>(P, n_shards, rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp, ln_nat);
}

int launch_rows_sum_ln(const float* P, int n_shards, int64_t rows, int64_t h, const void* bias,
                       const void* residual, const void* gamma, const void* beta, float eps,
                       void* Y_sum, void* Y_ln, cudaStream_t s, int sp_n, int sp_batch,
                       int sp_seq, int ln_natural) {
  if (rows <= 0) return 0;
  const SeqShard sp{sp_n, sp_batch, sp_seq};
  const int64_t nch = h / 8;
  if (n_shards == 0 && nch <= 32 * 32) {
    if (nch <= 32) launch_ln_warp<1>(rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp, ln_natural);
    else if (nch <= 64) launch_ln_warp<2>(rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp, ln_natural);
    else if (nch <= 128) launch_ln_warp<4>(rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp, ln_natural);
    else if (nch <= 256) launch_ln_warp<8>(rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp, ln_natural);
    else if (nch <= 512) launch_ln_warp<16>(rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp, ln_natural);
    else launch_ln_warp<32>(rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp, ln_natural);
  } else if (n_shards == 0)
    launch_rows<128>(P, n_shards, rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp,
                     ln_natural);
  else
    launch_rows<256>(P, n_shards, rows, h, bias, residual, gamma, beta, eps, Y_sum, Y_ln, s, sp,
                     ln_natural);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

int launch_all_gather_sequence(const void* Xs, int sp_n, int sp_batch, int sp_seq, int64_t h,
                               void* X, cudaStream_t s, int num_sms) {
  const SeqShard sp{sp_n, sp_batch, sp_seq};
  const int64_t n = static_cast<int64_t>(sp_batch) * sp_seq * h;
  int64_t blocks = (n / 8 + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  all_gather_sequence_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint16_t*>(Xs),
                                                     static_cast<uint16_t*>(X), n,
                                                     static_cast<int>(h), sp);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
