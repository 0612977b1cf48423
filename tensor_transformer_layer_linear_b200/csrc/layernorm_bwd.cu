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
//
// Rows of up to 8192 columns (rows_sum_ln_bwd_stream_kernel): one persistent
// CTA per SM walks rows strided over the grid. A producer warp streams the
// partials through a ring of 16 KB shared-memory stages with bulk copies
// (one stage = up to 4096 columns of one shard's row), so the next rows'
// partials are in flight while the consumers reduce the current one; 256
// consumer threads own 4-column groups (quads) of the row, add the stages
// into g in shard order, and take all four row statistics in one block
// reduction (sums of d = x - x[0], d^2, g gamma and g gamma d; the shift by
// the row's first element keeps E[d^2] - E[d]^2 well conditioned). The
// column sums of g x_hat and g stay in the consumers' registers; each CTA
// writes them once and a second pass adds the CTAs' sums in a fixed order,
// so dgamma and dbeta are deterministic.
// Wider rows (rows_sum_ln_bwd_kernel): one CTA of 256 threads per row at a
// time, 8 columns per thread per chunk, four block reductions per row, the
// column sums in shared memory.
// With a sequence-shard map (sequence parallelism) the partials stay in
// token order while x, the residual gradient and dx use the sequence-sharded
// layout: the reduce-scatter of the backward.
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

// ------------------------------------------------------- streamed variant
constexpr int kLnsConsumers = 256;                 // 8 consumer warps
constexpr int kLnsThreads = kLnsConsumers + 32;    // + the producer warp
constexpr int kLnsStageFloats = 4096;              // one stage: 16 KB
constexpr int kLnsStages = 12;
constexpr int kLnsStageQuads = kLnsStageFloats / 4;
constexpr int kLnsQuadsPerStage = kLnsStageQuads / kLnsConsumers;  // per thread
constexpr int kLnsMaxQuads = 8;                    // rows of up to 8192 columns
constexpr size_t kLnsSmem = static_cast<size_t>(kLnsStages) * kLnsStageFloats * 4 +
                            2 * kLnsStages * 8 + 2 * 8 * 16 + 16;

// bulk_load with an L2 eviction-priority policy (createpolicy)
__device__ __forceinline__ void bulk_load_evict_first(uint32_t dst, const void* src,
                                                      uint32_t bytes, uint32_t bar,
                                                      uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void lns_consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kLnsConsumers) : "memory");
}

__device__ __forceinline__ void unpack4(const uint2& b, float (&a)[4]) {
  a[0] = bf16_lo(b.x); a[1] = bf16_hi(b.x);
  a[2] = bf16_lo(b.y); a[3] = bf16_hi(b.y);
}

// KQ = quads (4-column groups) per consumer thread: thread t owns the
// row's quads t + 256 k (k < KQ); a stage carries 1024 quads, so quad k of
// a thread arrives in segment k / 4.
template <int KQ>
__global__ void __launch_bounds__(kLnsThreads, 1) rows_sum_ln_bwd_stream_kernel(
    const float* __restrict__ P, int n_shards, int64_t stride, int64_t rows, int h,
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ gamma,
    const uint16_t* __restrict__ res, float eps, uint16_t* __restrict__ dx,
    float* __restrict__ dg_part, float* __restrict__ db_part, SeqShard sp, unsigned* err) {
  constexpr int kSeg = (KQ + kLnsQuadsPerStage - 1) / kLnsQuadsPerStage;
  extern __shared__ __align__(128) unsigned char lns_smem[];
  float* ring = reinterpret_cast<float*>(lns_smem);
  const uint32_t bar0 = smem_u32(lns_smem + static_cast<size_t>(kLnsStages) * kLnsStageFloats * 4);
  auto full = [&](int st) { return bar0 + 8u * st; };
  auto empty = [&](int st) { return bar0 + 8u * (kLnsStages + st); };
  float4(*red4)[8] = reinterpret_cast<float4(*)[8]>(lns_smem + static_cast<size_t>(kLnsStages) *
                                                                    kLnsStageFloats * 4 +
                                                    2 * kLnsStages * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red4 + 2);
  const int quads = h >> 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kLnsStages; ++i) {
      mbar_init(full(i), 1);
      mbar_init(empty(i), kLnsConsumers / 32);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kLnsConsumers / 32) {
    // producer: one thread issues every stage's bulk copy, in the order the
    // consumers take them (row, segment, shard)
    if (lane != 0) return;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int used = 0;  // stages that received at least one copy
    // the partials are read once: let their lines go first from L2
    uint64_t policy;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
    for (int64_t r = blockIdx.x; r < rows && ok; r += gridDim.x) {
      for (int seg = 0; seg < kSeg && ok; ++seg) {
        const int q0 = seg * kLnsStageQuads;
        if (q0 >= quads) break;  // (the consumers skip the same segments)
        const int nq = min(kLnsStageQuads, quads - q0);
        for (int i = 0; i < n_shards; ++i) {
          if (!mbar_wait(empty(stage), phase ^ 1u, abort_flag)) {
            atomicOr(err, ERR_WAIT_PRODUCER);
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t bytes = static_cast<uint32_t>(nq) * 16u;
          mbar_arrive_expect_tx(full(stage), bytes);
          bulk_load_evict_first(smem_u32(ring + static_cast<size_t>(stage) * kLnsStageFloats),
                                P + i * stride + r * h + q0 * 4, bytes, full(stage), policy);
          if (used < kLnsStages) ++used;
          if (++stage == kLnsStages) { stage = 0; phase ^= 1u; }
        }
      }
    }
    // before the CTA may exit, every copy it issued has landed: the last
    // copy into stage st completed phase (st < stage ? phase : phase ^ 1)
    for (int st = 0; st < used; ++st) {
      const uint32_t last = st < stage ? phase : phase ^ 1u;
      int never = 0;
      if (!mbar_wait_for(full(st), last, &never, 100000000ull)) atomicOr(err, ERR_WAIT_PRODUCER);
    }
    return;
  }

  // consumers
  const int t = threadIdx.x;
  const float inv_h = 1.0f / static_cast<float>(h);
  // gamma stays in registers for rows of up to 4096 columns; wider rows
  // re-read it (L1) where it is used, to stay within the register budget
  constexpr bool kGammaRegs = KQ <= 4;
  uint2 gq[kGammaRegs ? KQ : 1];
  auto gamma_quad = [&](int k, int q) {
    return kGammaRegs ? gq[kGammaRegs ? k : 0] : __ldg(reinterpret_cast<const uint2*>(gamma) + q);
  };
  float cg[KQ][4], cb[KQ][4];
#pragma unroll
  for (int k = 0; k < KQ; ++k) {
    const int q = t + k * kLnsConsumers;
    if (kGammaRegs)
      gq[kGammaRegs ? k : 0] =
          q < quads ? __ldg(reinterpret_cast<const uint2*>(gamma) + q) : make_uint2(0u, 0u);
#pragma unroll
    for (int j = 0; j < 4; ++j) cg[k][j] = cb[k][j] = 0.f;
  }
  int stage = 0;
  uint32_t phase = 0;
  bool ok = true;
  int parity = 0;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x, parity ^= 1) {
    const int64_t soff = seq_shard_row(sp, r) * h;  // x, residual, dx
    // this row's x and residual gradient, in flight while the partials arrive
    uint2 xq[KQ], rq[KQ];
#pragma unroll
    for (int k = 0; k < KQ; ++k) {
      const int q = t + k * kLnsConsumers;
      xq[k] = rq[k] = make_uint2(0u, 0u);
      if (q < quads) {
        xq[k] = __ldg(reinterpret_cast<const uint2*>(x + soff) + q);
        if (res != nullptr) rq[k] = __ldg(reinterpret_cast<const uint2*>(res + soff) + q);
      }
    }
    const float piv = __uint_as_float(static_cast<uint32_t>(__ldg(x + soff)) << 16);
    // g = sum of the partials in shard order
    float g[KQ][4];
#pragma unroll
    for (int k = 0; k < KQ; ++k)
#pragma unroll
      for (int j = 0; j < 4; ++j) g[k][j] = 0.f;
#pragma unroll
    for (int seg = 0; seg < kSeg; ++seg) {
      if (seg * kLnsStageQuads >= quads) break;
      for (int i = 0; i < n_shards; ++i) {
        // after a failed wait (or another role's) the thread keeps its
        // barrier schedule without waiting; the result is discarded
        if (ok && !mbar_wait(full(stage), phase, abort_flag)) {
          ok = false;
          if (lane == 0) atomicOr(err, ERR_WAIT_EPILOGUE);
          *abort_flag = 1;
        }
        const float4* sv = reinterpret_cast<const float4*>(ring + static_cast<size_t>(stage) * kLnsStageFloats);
#pragma unroll
        for (int kk = 0; kk < kLnsQuadsPerStage; ++kk) {
          const int k = seg * kLnsQuadsPerStage + kk;
          if (k < KQ && t + k * kLnsConsumers < quads) {
            const float4 v = sv[t + kk * kLnsConsumers];
            g[k][0] += v.x; g[k][1] += v.y; g[k][2] += v.z; g[k][3] += v.w;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(stage));
        if (++stage == kLnsStages) { stage = 0; phase ^= 1u; }
      }
    }
    // the four row statistics in one block reduction
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < KQ; ++k) {
      if (t + k * kLnsConsumers < quads) {
        float xf[4], gm[4];
        unpack4(xq[k], xf);
        unpack4(gamma_quad(k, t + k * kLnsConsumers), gm);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float d = xf[j] - piv;
          const float gy = g[k][j] * gm[j];
          acc.x += d;
          acc.y += d * d;
          acc.z += gy;
          acc.w += gy * d;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
      acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
      acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
      acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
    }
    // two buffers alternate between rows: the next row's writes come after
    // every consumer passed the next barrier, so they never meet these reads
    if (lane == 0) red4[parity][warp] = acc;
    lns_consumer_sync();
    float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kLnsConsumers / 32; ++w) {
      const float4 a = red4[parity][w];
      tot.x += a.x; tot.y += a.y; tot.z += a.z; tot.w += a.w;
    }
    const float md = tot.x * inv_h;                       // mean - x[0]
    const float var = fmaxf(tot.y * inv_h - md * md, 0.f);
    const float rstd = rsqrtf(var + eps);
    const float m1 = tot.z * inv_h;                       // mean(g gamma)
    const float m2 = rstd * (tot.w * inv_h - md * m1);    // mean(g gamma x_hat)
#pragma unroll
    for (int k = 0; k < KQ; ++k) {
      const int q = t + k * kLnsConsumers;
      if (q < quads) {
        float xf[4], gm[4], rv[4], o[4];
        unpack4(xq[k], xf);
        unpack4(gamma_quad(k, t + k * kLnsConsumers), gm);
        unpack4(rq[k], rv);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float xh = (xf[j] - piv - md) * rstd;
          o[j] = rv[j] + rstd * (g[k][j] * gm[j] - m1 - xh * m2);
          cg[k][j] += g[k][j] * xh;
          cb[k][j] += g[k][j];
        }
        *(reinterpret_cast<uint2*>(dx + soff) + q) =
            make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
      }
    }
  }
#pragma unroll
  for (int k = 0; k < KQ; ++k) {
    const int q = t + k * kLnsConsumers;
    if (q < quads) {
      const int64_t o = static_cast<int64_t>(blockIdx.x) * h + 4 * q;
      *reinterpret_cast<float4*>(dg_part + o) = make_float4(cg[k][0], cg[k][1], cg[k][2], cg[k][3]);
      *reinterpret_cast<float4*>(db_part + o) = make_float4(cb[k][0], cb[k][1], cb[k][2], cb[k][3]);
    }
  }
}

template <int KQ>
static int launch_lns(const float* P, int n_shards, int64_t rows, int h, const void* x,
                      const void* gamma, const void* res, float eps, void* dx, float* dg_part,
                      float* db_part, int max_ctas, int num_sms, cudaStream_t s, SeqShard sp,
                      unsigned* err) {
  int ctas = num_sms;
  if (ctas > max_ctas) ctas = max_ctas;
  if (ctas > rows) ctas = static_cast<int>(rows);
  cudaFuncSetAttribute(rows_sum_ln_bwd_stream_kernel<KQ>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kLnsSmem));
  rows_sum_ln_bwd_stream_kernel<KQ><<<ctas, kLnsThreads, kLnsSmem, s>>>(
      P, n_shards, rows * h, rows, h, static_cast<const uint16_t*>(x),
      static_cast<const uint16_t*>(gamma), static_cast<const uint16_t*>(res), eps,
      static_cast<uint16_t*>(dx), dg_part, db_part, sp, err);
  return ctas;
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
                           cudaStream_t s, int num_sms, unsigned* err, int sp_n, int sp_batch,
                           int sp_seq) {
  if (rows <= 0) return 0;
  const SeqShard sp{sp_n, sp_batch, sp_seq};
  float* dg_part = part;
  float* db_part = part + static_cast<int64_t>(max_ctas) * h;
  const int hh = static_cast<int>(h);
  // quads per consumer thread, rounded up to 1, 2, 4 or 8 (the extra ones are
  // masked; up to four quads a row is one stage wide, five to eight two)
  const int64_t kq = (h / 4 + kLnsConsumers - 1) / kLnsConsumers;
  int ctas;
  if (kq <= 1)
    ctas = launch_lns<1>(P, n_shards, rows, hh, x, gamma, residual, eps, dx, dg_part, db_part, max_ctas, num_sms, s, sp, err);
  else if (kq <= 2)
    ctas = launch_lns<2>(P, n_shards, rows, hh, x, gamma, residual, eps, dx, dg_part, db_part, max_ctas, num_sms, s, sp, err);
  else if (kq <= 4)
    ctas = launch_lns<4>(P, n_shards, rows, hh, x, gamma, residual, eps, dx, dg_part, db_part, max_ctas, num_sms, s, sp, err);
  else if (kq <= kLnsMaxQuads)
    ctas = launch_lns<8>(P, n_shards, rows, hh, x, gamma, residual, eps, dx, dg_part, db_part, max_ctas, num_sms, s, sp, err);
  else
    ctas = launch_lnb_ch<8>(P, n_shards, rows, hh, x, gamma, residual, eps, dx, dg_part, db_part, max_ctas, num_sms, s, sp);
  if (launch_slab_sum(dg_part, ctas, hh, dgamma, s) != 0) return 2;
  if (launch_slab_sum(db_part, ctas, hh, dbeta, s) != 0) return 2;
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
