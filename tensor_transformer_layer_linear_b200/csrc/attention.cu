// Local self-attention of every shard's heads.
//
// "Tensor Parallelism in Large Language Models", "Local Self-Attention
// Computation": each GPU evaluates Head = softmax(Q K^T / sqrt(d_k)) V for
// its own heads with no communication. With the shards held on one GPU, one
// launch covers every (shard, sequence, local head, 128-query tile).
//
// Streaming (online) softmax over 64-key blocks, so memory is O(seq) and the
// S x S score matrix never exists: running row max m and row sum l in fp32,
// O rescaled by exp(m_old - m_new) when the max grows, divided by l at the
// end. Causal tiles stop at the diagonal, and heavy (late) query tiles are
// launched first. Q, K, V tiles are staged in XOR-swizzled shared memory
// with cp.async (double-buffered K/V); the two products run on the tensor
// cores through mma.sync m16n8k16 (bf16 in, fp32 accumulate), P is rounded to
// bf16 in registers for the second product.
#include <math.h>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

constexpr int AT_BM = 128;   // queries per CTA (8 warps x 16 rows)
constexpr int AT_BN = 64;    // keys per block
constexpr int AT_D = 128;    // head dim
constexpr int AT_THREADS = 256;
constexpr int AT_TILE_Q = AT_BM * AT_D * 2;   // 32 KB
constexpr int AT_TILE_KV = AT_BN * AT_D * 2;  // 16 KB
constexpr int AT_SMEM = AT_TILE_Q + 4 * AT_TILE_KV;

// byte offset of 16-byte chunk c (0..15) of row r in a [rows][128] bf16 tile
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * 256 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(AT_THREADS, 1)
    attention_fwd_kernel(const uint16_t* __restrict__ QKV, uint16_t* __restrict__ O, int seq,
                         int batch, int hps, int hs, int causal, float scale_log2,
                         int num_q_tiles) {
  extern __shared__ __align__(128) uint8_t sm[];
  const uint32_t sQ = smem_u32(sm);
  const uint32_t sK = sQ + AT_TILE_Q;
  const uint32_t sV = sK + 2 * AT_TILE_KV;

  const int qt = causal ? (num_q_tiles - 1 - static_cast<int>(blockIdx.x)) : blockIdx.x;
  const int y = blockIdx.y;
  const int head = y % hps;
  const int sidx = (y / hps) % batch;
  const int g = y / (hps * batch);
  const int64_t M = static_cast<int64_t>(batch) * seq;
  const int ld = 3 * hs;
  const uint16_t* base = QKV + (static_cast<int64_t>(g) * M + static_cast<int64_t>(sidx) * seq) * ld;
  const uint16_t* Qp = base + head * AT_D;
  const uint16_t* Kp = base + hs + head * AT_D;
  const uint16_t* Vp = base + 2 * hs + head * AT_D;
  const int q0 = qt * AT_BM;

  for (int i = threadIdx.x; i < AT_BM * 16; i += AT_THREADS) {
    const int r = i >> 4, c = i & 15;
    const bool v = q0 + r < seq;
    cp_async16(sQ + swz(r, c), Qp + static_cast<int64_t>(v ? q0 + r : 0) * ld + c * 8, v);
  }
  auto load_kv = [&](int j, int buf) {
    const int k0 = j * AT_BN;
    for (int i = threadIdx.x; i < AT_BN * 16; i += AT_THREADS) {
      const int r = i >> 4, c = i & 15;
      const bool v = k0 + r < seq;
      const int64_t off = static_cast<int64_t>(v ? k0 + r : 0) * ld + c * 8;
      cp_async16(sK + buf * AT_TILE_KV + swz(r, c), Kp + off, v);
      cp_async16(sV + buf * AT_TILE_KV + swz(r, c), Vp + off, v);
    }
  };
  load_kv(0, 0);
  cp_async_commit();
  int n_blocks = (seq + AT_BN - 1) / AT_BN;
  if (causal) {
    const int last = (q0 + AT_BM - 1) / AT_BN + 1;
    if (last < n_blocks) n_blocks = last;
  }
  cp_async_wait_all();
  __syncthreads();

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wr = warp * 16;

  uint32_t qf[8][4];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) ldsm_x4(qf[kk], sQ + swz(wr + (lane & 15), kk * 2 + (lane >> 4)));

  float o[16][4];
#pragma unroll
  for (int t = 0; t < 16; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
  const int row_a = q0 + wr + (lane >> 2);
  const int row_b = row_a + 8;

  for (int j = 0; j < n_blocks; ++j) {
    const int buf = j & 1;
    if (j + 1 < n_blocks) load_kv(j + 1, buf ^ 1);
    cp_async_commit();
    const int k0 = j * AT_BN;
    const bool skip = causal && (k0 > q0 + wr + 15);  // every key after every row of this warp
    if (!skip) {
      float s[8][4];
#pragma unroll
      for (int t = 0; t < 8; ++t) s[t][0] = s[t][1] = s[t][2] = s[t][3] = 0.f;
      const uint32_t kb = sK + buf * AT_TILE_KV;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
        for (int nt = 0; nt < 8; nt += 2) {
          uint32_t b[4];
          ldsm_x4(b, kb + swz(nt * 8 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)));
          mma_bf16_16816(s[nt], qf[kk], b[0], b[1]);
          mma_bf16_16816(s[nt + 1], qf[kk], b[2], b[3]);
        }
      }
      if (k0 + AT_BN > seq || (causal && k0 + AT_BN - 1 > q0 + wr)) {
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = k0 + nt * 8 + (lane & 3) * 2 + (e & 1);
            const int row = (e < 2) ? row_a : row_b;
            if (key >= seq || (causal && key > row)) s[nt][e] = -INFINITY;
          }
        }
      }
      float mx_a = m_a, mx_b = m_b;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        mx_a = fmaxf(mx_a, fmaxf(s[nt][0], s[nt][1]));
        mx_b = fmaxf(mx_b, fmaxf(s[nt][2], s[nt][3]));
      }
      mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
      mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
      mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
      mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
      const float base_a = (mx_a == -INFINITY) ? 0.f : mx_a * scale_log2;
      const float base_b = (mx_b == -INFINITY) ? 0.f : mx_b * scale_log2;
      const float alpha_a = exp2f(m_a * scale_log2 - base_a);
      const float alpha_b = exp2f(m_b * scale_log2 - base_b);
      m_a = mx_a;
      m_b = mx_b;
      float sum_a = 0.f, sum_b = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        s[nt][0] = exp2f(s[nt][0] * scale_log2 - base_a);
        s[nt][1] = exp2f(s[nt][1] * scale_log2 - base_a);
        s[nt][2] = exp2f(s[nt][2] * scale_log2 - base_b);
        s[nt][3] = exp2f(s[nt][3] * scale_log2 - base_b);
        sum_a += s[nt][0] + s[nt][1];
        sum_b += s[nt][2] + s[nt][3];
      }
      l_a = l_a * alpha_a + sum_a;
      l_b = l_b * alpha_b + sum_b;
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        o[t][0] *= alpha_a;
        o[t][1] *= alpha_a;
        o[t][2] *= alpha_b;
        o[t][3] *= alpha_b;
      }
      const uint32_t vb = sV + buf * AT_TILE_KV;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t a[4];
        a[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
        a[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
        a[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        a[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int nt = 0; nt < 16; nt += 2) {
          uint32_t b[4];
          ldsm_x4_t(b, vb + swz(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), nt + (lane >> 4)));
          mma_bf16_16816(o[nt], a, b[0], b[1]);
          mma_bf16_16816(o[nt + 1], a, b[2], b[3]);
        }
      }
    }
    cp_async_wait_all();
    __syncthreads();
  }

  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  const float inv_a = l_a > 0.f ? 1.f / l_a : 0.f;
  const float inv_b = l_b > 0.f ? 1.f / l_b : 0.f;

  // Stage this warp's 16 output rows in its own rows of the Q tile, then
  // write them out with 16-byte stores.
  const int ra = wr + (lane >> 2), rb = ra + 8;
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const uint32_t off = static_cast<uint32_t>((lane & 3) * 4);
    const uint32_t va = pack_bf16x2(o[nt][0] * inv_a, o[nt][1] * inv_a);
    const uint32_t vbv = pack_bf16x2(o[nt][2] * inv_b, o[nt][3] * inv_b);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(sQ + swz(ra, nt) + off), "r"(va) : "memory");
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(sQ + swz(rb, nt) + off), "r"(vbv) : "memory");
  }
  __syncwarp();
  uint16_t* Ob = O + (static_cast<int64_t>(g) * M + static_cast<int64_t>(sidx) * seq) * hs + head * AT_D;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int i = lane + 32 * it;
    const int r = i >> 4, c = i & 15;
    const int qrow = q0 + wr + r;
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(sQ + swz(wr + r, c)));
    if (qrow < seq) *reinterpret_cast<uint4*>(Ob + static_cast<int64_t>(qrow) * hs + c * 8) = v;
  }
}

int launch_attention(const void* QKV, int64_t batch, int64_t seq, int64_t h, int64_t n_heads,
                     int n_shards, int causal, void* O, cudaStream_t s, unsigned* err) {
  (void)err;
  const int hps = static_cast<int>(n_heads / n_shards);
  const int hs = static_cast<int>(h / n_shards);
  const int nq = static_cast<int>((seq + AT_BM - 1) / AT_BM);
  cudaFuncSetAttribute(attention_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM);
  const dim3 grid(nq, static_cast<unsigned>(n_shards * batch * hps));
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(h / n_heads));
  attention_fwd_kernel<<<grid, AT_THREADS, AT_SMEM, s>>>(
      static_cast<const uint16_t*>(QKV), static_cast<uint16_t*>(O), static_cast<int>(seq),
      static_cast<int>(batch), hps, hs, causal, scale_log2, nq);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
