// Local self-attention of every shard's heads on the 5th-generation tensor
// cores.
//
// "Tensor Parallelism in Large Language Models", "Local Self-Attention
// Computation": each GPU evaluates Head = softmax(Q K^T / sqrt(d_k)) V for
// its own heads with no communication. With the shards held on one GPU, one
// launch covers every (shard, sequence, local head, 128-query tile).
//
// One CTA per 128-query tile (d = 128), 8 warps:
//   warps 0-3  softmax: one thread per query row (= TMEM lane). The row of S
//              is read from TMEM into registers, masked on diagonal / tail
//              blocks, its max taken, P = exp2(S scale - m) formed in fp32
//              with the row sum, and P stored as bf16 pairs back into TMEM
//              over the S columns. The running max moves lazily: O and the
//              sum are rescaled only when the max grows by more than 2^8, so
//              P stays <= 256 and O / l is unchanged (the same max scales
//              numerator and denominator).
//   warp 4     TMA: the Q tile once, then 128-key K blocks into a 2-deep ring
//              straight out of the QKV projection's [shard][token][3h/N]
//              output (128-byte swizzle).
//   warp 6     TMA: the V blocks into their own 2-deep ring.
//   warp 5     TMEM owner and the single MMA-issuing thread.
// S is double-buffered in TMEM, so the MMAs of a key block overlap the
// softmax of the previous one. MMA issue order:
//   S_0 = Q K_0^T | S_1 = Q K_1^T | O = P_0 V_0 | S_2 = Q K_2^T |
//   O += P_1 V_1 | S_3 = Q K_3^T | ...
// S_{j+2} overwrites the buffer holding P_j right after the MMA that reads
// it, relying on one thread's tcgen05.mma operations executing in issue
// order. A commit after every PV tells the softmax when O holds exactly the
// blocks before its own (needed only for a rescale).
// TMEM: S / P buffer b at columns [128 b, 128 b + 128), O at [256, 384).
// Causal CTAs stop at their diagonal block; heavy (late) query tiles launch
// first. Every barrier wait is bounded; a role that gives up records an
// error bit and the CTA leaves through the common exit after waiting
// (bounded) for its copies and MMAs in flight.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

constexpr int FA_BM = 128;                  // queries per tile (one tile per CTA)
constexpr int FA_BN = 128;                  // keys per block
constexpr int FA_D = 128;                   // head dim
constexpr int FA_THREADS = 256;             // 8 warps: up to 255 registers per thread
constexpr int FA_SUB = 128 * 128;           // one [128 rows][64 cols] bf16 box: 16 KB
constexpr int FA_TILE = 2 * FA_SUB;         // a [128][128] bf16 tile: 32 KB
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + FA_TILE;      // 2 buffers
constexpr int OFF_V = OFF_K + 2 * FA_TILE;  // 2 buffers
constexpr int OFF_BAR = OFF_V + 2 * FA_TILE;
constexpr int FA_NUM_BARS = 16;
constexpr int FA_SMEM = 1024 + OFF_BAR + FA_NUM_BARS * 8 + 16;
static_assert(FA_SMEM <= 232448, "shared memory budget");

// barrier indices (K, V, S and P per buffer b)
constexpr int B_Q = 0, B_KFULL = 1, B_VFULL = 3, B_KEMPTY = 5, B_VEMPTY = 7, B_SFULL = 9,
              B_PFULL = 11, B_OUPD = 13, B_ODONE = 14;

struct AttnParams {
  int seq, batch, hps, causal, nq;
  int q_w;    // query columns per shard (query heads per shard x 128)
  int kv_w;   // key (= value) columns per shard
  int group;  // local query heads per local kv head
  long long M;  // tokens per shard
  float scale_log2;
  float* lse;  // optional: base-2 log-sum-exp of each query's scaled scores
  long long lse_stride;  // per (shard, head): tokens per shard + 128
  unsigned* err;
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__global__ void __launch_bounds__(FA_THREADS, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm, uint16_t* __restrict__ O,
                        const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* sm = smem_raw + pad;
  const uint32_t s0 = smem_u32(sm);
  const uint32_t bar0 = s0 + OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + OFF_BAR + FA_NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = p.causal ? (p.nq - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x);
  const int y = blockIdx.y;
  const int head = y % p.hps;
  const int sidx = (y / p.hps) % p.batch;
  const int g = y / (p.hps * p.batch);
  const int q0 = qt * FA_BM;
  const int row_base = sidx * p.seq;  // first token of this sequence within the shard
  int nb = (p.seq + FA_BN - 1) / FA_BN;
  if (p.causal) {
    const int last = (q0 + FA_BM - 1) / FA_BN + 1;
    if (last < nb) nb = last;
  }
  const int kvh = head / p.group;  // this query head's local kv head
  const int kcol = p.q_w + kvh * FA_D, vcol = p.q_w + p.kv_w + kvh * FA_D;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_KFULL + b), 1);
      mbar_init(bar(B_VFULL + b), 1);
      mbar_init(bar(B_KEMPTY + b), 1);
      mbar_init(bar(B_VEMPTY + b), 1);
      mbar_init(bar(B_SFULL + b), 1);
      mbar_init(bar(B_PFULL + b), 4);  // one arrival per softmax warp
    }
    mbar_init(bar(B_OUPD), 1);
    mbar_init(bar(B_ODONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) tma_prefetch_desc(&tm);
  if (warp == 5) tmem_alloc(smem_u32(tmem_holder), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 4 || warp == 6) {
    // ------------------------------------------------------------ TMA (Q + K | V)
    if (lane == 0) {
      const bool is_k = warp == 4;
      const int col = is_k ? kcol : vcol;
      const int full = is_k ? B_KFULL : B_VFULL, empty = is_k ? B_KEMPTY : B_VEMPTY;
      const uint32_t ring = s0 + (is_k ? OFF_K : OFF_V);
      bool ok = true;
      if (is_k) {
        mbar_arrive_expect_tx(bar(B_Q), FA_TILE);
        const int qrow = row_base + q0;
        tma_load_3d(s0 + OFF_Q, &tm, bar(B_Q), head * FA_D, qrow, g);
        tma_load_3d(s0 + OFF_Q + FA_SUB, &tm, bar(B_Q), head * FA_D + 64, qrow, g);
      }
      int issued = 0;
      for (int j = 0; j < nb; ++j) {
        const int b = j & 1;
        if (!mbar_wait(bar(empty + b), ((j >> 1) & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t d = ring + b * FA_TILE;
        const int krow = row_base + j * FA_BN;
        mbar_arrive_expect_tx(bar(full + b), FA_TILE);
        tma_load_3d(d, &tm, bar(full + b), col, krow, g);
        tma_load_3d(d + FA_SUB, &tm, bar(full + b), col + 64, krow, g);
        ++issued;
      }
      if (!ok) {
        atomicOr(p.err, ERR_WAIT_ATTN);
        *abort_flag = 1;
      }
      // every load issued must land before the CTA exits
      int never = 0;
      if (is_k && !mbar_wait(bar(B_Q), 0, &never)) atomicOr(p.err, ERR_WAIT_DRAIN);
      for (int jj = (issued >= 2 ? issued - 2 : 0); jj < issued; ++jj)
        if (!mbar_wait(bar(full + (jj & 1)), (jj >> 1) & 1, &never))
          atomicOr(p.err, ERR_WAIT_DRAIN);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16_f32(FA_BM, FA_BN);
      constexpr uint32_t idesc_o = umma_idesc_bf16_f32_bmn(FA_BM, FA_D);
      // descriptors built once; each MMA moves them by a constant offset
      const uint64_t dq = umma_desc_sw128(s0 + OFF_Q);
      const uint64_t dk0 = umma_desc_sw128(s0 + OFF_K), dk1 = umma_desc_sw128(s0 + OFF_K + FA_TILE);
      const uint64_t dv0 = umma_desc_sw128_mn(s0 + OFF_V, FA_SUB);
      const uint64_t dv1 = umma_desc_sw128_mn(s0 + OFF_V + FA_TILE, FA_SUB);
      // S_j = Q K_j^T into buffer j & 1
      auto qk = [&](int j) -> bool {
        const int b = j & 1;
        if (!mbar_wait(bar(B_KFULL + b), (j >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dk = b ? dk1 : dk0;
#pragma unroll
        for (int kk = 0; kk < FA_D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * FA_SUB + (kk & 3) * 32;
          umma_bf16(tmem + b * FA_BN, desc_advance(dq, off), desc_advance(dk, off), idesc_s,
                    kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(B_KEMPTY + b));
        umma_commit(bar(B_SFULL + b));
        return true;
      };
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag);
      if (ok) ok = qk(0);
      if (ok && nb > 1) ok = qk(1);
      for (int j = 0; ok && j < nb; ++j) {
        const int b = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(bar(B_VFULL + b), ph, abort_flag) ||
            !mbar_wait(bar(B_PFULL + b), ph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t dv = b ? dv1 : dv0;
#pragma unroll
        for (int kk = 0; kk < FA_BN / 16; ++kk)             // O (+)= P_j V_j
          umma_bf16_tmem_a(tmem + 2 * FA_BN, tmem + b * FA_BN + kk * 8,
                           desc_advance(dv, kk * 2048), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(B_VEMPTY + b));
        umma_commit(bar(B_OUPD));
        if (j + 2 < nb) ok = qk(j + 2);                    // reuses the buffer P_j was in
      }
      if (!ok) {
        atomicOr(p.err, ERR_WAIT_ATTN);
        *abort_flag = 1;
      }
      // o_done doubles as the drain of every MMA this thread issued
      umma_commit(bar(B_ODONE));
      int never = 0;
      if (!mbar_wait(bar(B_ODONE), 0, &never)) atomicOr(p.err, ERR_WAIT_DRAIN);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ softmax
    const int r = warp * 32 + lane;  // row within the tile (= TMEM lane)
    const int t = q0 + r;            // query position within the sequence
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t o_cols = tmem + lane_addr + 2 * FA_BN;
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nb; ++j) {
      const int b = j & 1;
      if (!mbar_wait(bar(B_SFULL + b), (j >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_cols = tmem + lane_addr + b * FA_BN;
      const int k0 = j * FA_BN;
      uint32_t v[FA_BN];
#pragma unroll
      for (int c = 0; c < FA_BN / 32; ++c) tmem_ld_32x32b_x32(s_cols + c * 32, &v[c * 32]);
      tmem_ld_wait();
      if (k0 + FA_BN > p.seq || (p.causal && k0 + FA_BN - 1 > q0)) {
        // keys k0 + e with e >= lim are past the sequence or (causal) after t
        const int lim = min(p.seq, p.causal ? t + 1 : p.seq) - k0;
#pragma unroll
        for (int e = 0; e < FA_BN; ++e) v[e] = e < lim ? v[e] : 0xFF800000u;  // -inf
      }
      float m8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) m8[u] = fmaxf(__uint_as_float(v[u]), __uint_as_float(v[u + 8]));
#pragma unroll
      for (int e = 16; e < FA_BN; e += 16) {
#pragma unroll
        for (int u = 0; u < 8; ++u)
          m8[u] = fmax3(m8[u], __uint_as_float(v[e + u]), __uint_as_float(v[e + 8 + u]));
      }
      const float mx = fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
      // lazy max: move it (and rescale) only when exp2 would exceed 2^8
      const bool need = (mx != -INFINITY) && ((mx - m_used) * sl2 > 8.f);
      float alpha = 1.f;
      if (need) {
        alpha = exp2f((m_used - mx) * sl2);  // 0 when m_used is still -inf
        l *= alpha;
        m_used = mx;
      }
      if (__any_sync(0xffffffffu, need && j > 0)) {
        // O must hold exactly the blocks before j: wait for PV_{j-1}
        if (!mbar_wait(bar(B_OUPD), (j - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < FA_D / 32; ++c) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(o_cols + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st_32x32b_x32(o_cols + c * 32, o);
        }
      }
      const float base = (m_used == -INFINITY) ? 0.f : m_used * sl2;
      float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < FA_BN / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float a = ex2_approx(fmaf(__uint_as_float(v[c * 32 + e]), sl2, -base));
          const float bb = ex2_approx(fmaf(__uint_as_float(v[c * 32 + e + 1]), sl2, -base));
          s8[(e >> 1) & 7] += a + bb;
          pk[e >> 1] = pack_bf16x2(a, bb);
        }
        tmem_st_32x32b_x16(s_cols + c * 16, pk);
      }
      l += ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_PFULL + b));
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, ERR_WAIT_ATTN);
      *abort_flag = 1;
    } else if (mbar_wait(bar(B_ODONE), 0, abort_flag)) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float base_final = (m_used == -INFINITY) ? 0.f : m_used * sl2;
      uint16_t* orow = O + (static_cast<int64_t>(g) * p.M + row_base + t) * p.q_w + head * FA_D;
#pragma unroll 1
      for (int c = 0; c < FA_D / 32; ++c) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(o_cols + c * 32, o);
        tmem_ld_wait();
        if (t < p.seq) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * e + 0]) * inv, __uint_as_float(o[8 * e + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + 8 * e) = w;
          }
        }
      }
      // P = exp2(s sl2 - base) / l = exp2(s sl2 - (base + log2 l))
      if (p.lse != nullptr && t < p.seq)
        p.lse[(static_cast<int64_t>(g) * p.hps + head) * p.lse_stride + row_base + t] =
            base_final + log2f(l);
    } else {
      if (lane == 0) atomicOr(p.err, ERR_WAIT_ATTN);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 attn_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

int launch_attention(const void* QKV, int64_t batch, int64_t seq, int64_t n_q, int64_t kv_local,
                     int n_shards, int causal, void* O, cudaStream_t s, unsigned* err,
                     float* lse) {
  const int hps = static_cast<int>(n_q / n_shards);
  const int64_t q_w = hps * FA_D, kv_w = kv_local * FA_D;
  const int64_t ld = q_w + 2 * kv_w;  // QKV row width per shard
  const int64_t M = batch * seq;
  auto enc = attn_map_encoder();
  if (enc == nullptr) return 1;
  CUtensorMap tm;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(ld), static_cast<cuuint64_t>(M),
                        static_cast<cuuint64_t>(n_shards)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld * 2), static_cast<cuuint64_t>(M * ld * 2)};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(QKV), dims, strides, box,
          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return 1;
  AttnParams p;
  p.seq = static_cast<int>(seq);
  p.batch = static_cast<int>(batch);
  p.hps = hps;
  p.q_w = static_cast<int>(q_w);
  p.kv_w = static_cast<int>(kv_w);
  p.group = static_cast<int>(hps / kv_local);
  p.causal = causal;
  p.nq = static_cast<int>((seq + FA_BM - 1) / FA_BM);
  p.M = M;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(FA_D));
  p.lse = lse;
  p.lse_stride = M + 128;
  p.err = err;
  cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, FA_SMEM);
  const dim3 grid(p.nq, static_cast<unsigned>(n_shards * batch * hps));
  attention_tc_kernel<<<grid, FA_THREADS, FA_SMEM, s>>>(tm, static_cast<uint16_t*>(O), p);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
