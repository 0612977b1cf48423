// The backward reduction of a pre-LN block: the block's one all-reduce (the
// sum of the N partial input gradients, "Tensor Parallelism in Large Language
// Models", "Communication Budget and Scaling Limits") fused with the
// LayerNorm backward and the residual path that bypasses the block.
//
// For a row with LN input x (mean mu, population variance var, rstd =
// 1 / sqrt(var + eps)), x_hat = (x - mu) rstd, and g = sum_i P_i the gradient
// reaching the LN output:
//   dx = R + rstd (g gamma - mean(g gamma) - x_hat mean(g gamma x_hat)),
//   dgamma += g x_hat,  dbeta += g   (summed over rows).
// One CTA of 256 threads per row at a time (rows strided over the grid), 8
// columns per thread per chunk, fp32 statistics of the bf16 input, four
// block reductions per row. Each CTA keeps its column sums of g x_hat and g
// in shared memory (every column owned by one thread) and writes them once;
// a second pass adds the CTAs' sums in a fixed order, so dgamma and dbeta
// are deterministic. With a sequence-shard map (sequence parallelism) the
// partials stay in token order while x, the residual gradient and dx use the
// sequence-sharded layout: the reduce-scatter of the backward.
#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

constexpr int kLnbThreads = 256;

template <int T>
__device__ __forceinline__ float lnb_block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < T / 32; ++i) t += red[i];
  __syncthreads();
  return t;
}

__device__ __forceinline__ void unpack8(const uint4& b, float (&a)[8]) {
  a[0] = bf16_lo(b.x); a[1] = bf16_hi(b.x);
  a[2] = bf16_lo(b.y); a[3] = bf16_hi(b.y);
  a[4] = bf16_lo(b.z); a[5] = bf16_hi(b.z);
  a[6] = bf16_lo(b.w); a[7] = bf16_hi(b.w);
}

template <int CH, int NS>
__global__ void __launch_bounds__(kLnbThreads, (CH <= 2 ? 3 : 1)) rows_sum_ln_bwd_kernel(
    const float* __restrict__ P, int n_shards, int64_t stride, int64_t rows, int h,
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ gamma,
    const uint16_t* __restrict__ res, float eps, uint16_t* __restrict__ dx,
    float* __restrict__ dg_part, float* __restrict__ db_part, SeqShard sp) {
  __shared__ float red[kLnbThreads / 32];
  extern __shared__ float colsums[];  // [2][h]: sums of g x_hat, then of g
  const int nch = h >> 3;
  const float inv_h = 1.0f / static_cast<float>(h);
  for (int c = threadIdx.x; c < 2 * h; c += kLnbThreads) colsums[c] = 0.f;
  // (the barriers of the first row's block reductions order this before any
  // thread adds to its columns; every CTA has at least one row)
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const int64_t off = r * h;                      // partials: token order
    const int64_t soff = seq_shard_row(sp, r) * h;  // x, residual, dx
    float xv[CH][8], gv[CH][8], gm[CH][8];
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = threadIdx.x + c * kLnbThreads;
      if (ch < nch) {
        const int64_t e = off + (ch << 3);
        unpack8(__ldg(reinterpret_cast<const uint4*>(x + soff + (ch << 3))), xv[c]);
        // the gradient reaching the LN output: sum of the partials in shard order
        if constexpr (NS > 0) {
          float4 v[NS][2];
#pragma unroll
          for (int i = 0; i < NS; ++i) {
            const float4* src = reinterpret_cast<const float4*>(P + i * stride + e);
            v[i][0] = __ldcs(src);
            v[i][1] = __ldcs(src + 1);
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) gv[c][j] = 0.f;
#pragma unroll
          for (int i = 0; i < NS; ++i) {
            gv[c][0] += v[i][0].x; gv[c][1] += v[i][0].y; gv[c][2] += v[i][0].z;
            gv[c][3] += v[i][0].w; gv[c][4] += v[i][1].x; gv[c][5] += v[i][1].y;
            gv[c][6] += v[i][1].z; gv[c][7] += v[i][1].w;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) gv[c][j] = 0.f;
          for (int i = 0; i < n_shards; ++i) {
            const float4* src = reinterpret_cast<const float4*>(P + i * stride + e);
            const float4 a = __ldcs(src), b = __ldcs(src + 1);
            gv[c][0] += a.x; gv[c][1] += a.y; gv[c][2] += a.z; gv[c][3] += a.w;
            gv[c][4] += b.x; gv[c][5] += b.y; gv[c][6] += b.z; gv[c][7] += b.w;
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) s += xv[c][j];
        unpack8(__ldg(reinterpret_cast<const uint4*>(gamma + (ch << 3))), gm[c]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) xv[c][j] = gv[c][j] = gm[c][j] = 0.f;
      }
    }
    const float mean = lnb_block_sum<kLnbThreads>(s, red) * inv_h;
    float q = 0.f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = threadIdx.x + c * kLnbThreads;
      if (ch < nch) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float d = xv[c][j] - mean;
          q += d * d;
        }
      }
    }
    const float rstd = rsqrtf(lnb_block_sum<kLnbThreads>(q, red) * inv_h + eps);
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        xv[c][j] = (xv[c][j] - mean) * rstd;       // x_hat
        const float gy = gv[c][j] * gm[c][j];      // g gamma (0 past the row)
        s1 += gy;
        s2 += gy * xv[c][j];
      }
    }
    const float m1 = lnb_block_sum<kLnbThreads>(s1, red) * inv_h;
    const float m2 = lnb_block_sum<kLnbThreads>(s2, red) * inv_h;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int ch = threadIdx.x + c * kLnbThreads;
      if (ch < nch) {
        const int64_t e = soff + (ch << 3);
        float rv[8];
        if (res != nullptr) {
          unpack8(__ldg(reinterpret_cast<const uint4*>(res + e)), rv);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) rv[j] = 0.f;
        }
        float o[8];
        float* cg = colsums + (ch << 3);
        float* cb = colsums + h + (ch << 3);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          o[j] = rv[j] + rstd * (gv[c][j] * gm[c][j] - m1 - xv[c][j] * m2);
          cg[j] += gv[c][j] * xv[c][j];
          cb[j] += gv[c][j];
        }
        uint4 w;
        w.x = pack_bf16x2(o[0], o[1]);
        w.y = pack_bf16x2(o[2], o[3]);
        w.z = pack_bf16x2(o[4], o[5]);
        w.w = pack_bf16x2(o[6], o[7]);
        *reinterpret_cast<uint4*>(dx + e) = w;
      }
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < h; c += kLnbThreads) {
    dg_part[static_cast<int64_t>(blockIdx.x) * h + c] = colsums[c];
    db_part[static_cast<int64_t>(blockIdx.x) * h + c] = colsums[h + c];
  }
}

// CTAs resident per SM: three for rows of up to 4096 columns (register
// budget), else one
template <int CH>
constexpr int lnb_ctas_per_sm() {
  return CH <= 2 ? 3 : 1;
}

template <int CH>
static int launch_lnb_ch(const float* P, int n_shards, int64_t rows, int h, const void* x,
                         const void* gamma, const void* res, float eps, void* dx, float* dg_part,
                         float* db_part, int max_ctas, int num_sms, cudaStream_t s,
                         SeqShard sp) {
  int ctas = lnb_ctas_per_sm<CH>() * num_sms;
  if (ctas > max_ctas) ctas = max_ctas;
  if (ctas > rows) ctas = static_cast<int>(rows);
  auto X = static_cast<const uint16_t*>(x);
  auto G = static_cast<const uint16_t*>(gamma);
  auto R = static_cast<const uint16_t*>(res);
  auto D = static_cast<uint16_t*>(dx);
  const int64_t stride = rows * h;
  const size_t smem = 2 * static_cast<size_t>(h) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaFuncSetAttribute(rows_sum_ln_bwd_kernel<CH, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    cudaFuncSetAttribute(rows_sum_ln_bwd_kernel<CH, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    cudaFuncSetAttribute(rows_sum_ln_bwd_kernel<CH, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    cudaFuncSetAttribute(rows_sum_ln_bwd_kernel<CH, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    cudaFuncSetAttribute(rows_sum_ln_bwd_kernel<CH, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  }
  switch (n_shards) {
    case 1: rows_sum_ln_bwd_kernel<CH, 1><<<ctas, kLnbThreads, smem, s>>>(P, 1, stride, rows, h, X, G, R, eps, D, dg_part, db_part, sp); break;
    case 2: rows_sum_ln_bwd_kernel<CH, 2><<<ctas, kLnbThreads, smem, s>>>(P, 2, stride, rows, h, X, G, R, eps, D, dg_part, db_part, sp); break;
    case 4: rows_sum_ln_bwd_kernel<CH, 4><<<ctas, kLnbThreads, smem, s>>>(P, 4, stride, rows, h, X, G, R, eps, D, dg_part, db_part, sp); break;
    case 8: rows_sum_ln_bwd_kernel<CH, 8><<<ctas, kLnbThreads, smem, s>>>(P, 8, stride, rows, h, X, G, R, eps, D, dg_part, db_part, sp); break;
    default: rows_sum_ln_bwd_kernel<CH, 0><<<ctas, kLnbThreads, smem, s>>>(P, n_shards, stride, rows, h, X, G, R, eps, D, dg_part, db_part, sp); break;
  }
  return ctas;
}

int launch_rows_sum_ln_bwd(const float* P, int n_shards, int64_t rows, int64_t h, const void* x,
                           const void* gamma, const void* residual, float eps, void* dx,
                           float* dgamma, float* dbeta, float* part, int max_ctas,
                           cudaStream_t s, int num_sms, int sp_n, int sp_batch, int sp_seq) {
  if (rows <= 0) return 0;
  const SeqShard sp{sp_n, sp_batch, sp_seq};
  float* dg_part = part;
  float* db_part = part + static_cast<int64_t>(max_ctas) * h;
  const int hh = static_cast<int>(h);
  const int64_t nch = h / 8;
  int ctas;
  if (nch <= kLnbThreads)
    ctas = launch_lnb_ch<1>(P, n_shards, rows, hh, x, gamma, residual, eps, dx, dg_part, db_part, max_ctas, num_sms, s, sp);
  else if (nch <= 2 * kLnbThreads)
    ctas = launch_lnb_ch<2>(P, n_shards, rows, hh, x, gamma, residual, eps, dx, dg_part, db_part, max_ctas, num_sms, s, sp);
  else if (nch <= 4 * kLnbThreads)
    ctas = launch_lnb_ch<4>(P, n_shards, rows, hh, x, gamma, residual, eps, dx, dg_part, db_part, max_ctas, num_sms, s, sp);
  else
    ctas = launch_lnb_ch<8>(P, n_shards, rows, hh, x, gamma, residual, eps, dx, dg_part, db_part, max_ctas, num_sms, s, sp);
  if (launch_slab_sum(dg_part, ctas, hh, dgamma, s) != 0) return 2;
  if (launch_slab_sum(db_part, ctas, hh, dbeta, s) != 0) return 2;
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
