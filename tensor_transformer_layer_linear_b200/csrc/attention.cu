// Local self-attention of every shard's heads on the 5th-generation tensor
// cores.
//
// "Tensor Parallelism in Large Language Models", "Local Self-Attention
// Computation": each GPU evaluates Head = softmax(Q K^T / sqrt(d_k)) V for
// its own heads with no communication. With the shards held on one GPU, one
// launch covers every (shard, sequence, local head, 128-query tile).
//
// One CTA per 128-query tile (d = 128), 6 warps:
//   warp 0     TMA: the Q tile once, then 128-key K and V blocks into a
//              2-deep ring (each block two 64-column boxes, 128-byte swizzle)
//              straight out of the QKV projection's [shard][token][3h/N]
//              output.
//   warp 1     one thread issues tcgen05.mma: S_j = Q K_j^T into one of two
//              TMEM score buffers (K-major A and B), then O += P_{j-1} V_{j-1}
//              into the TMEM output accumulator (P K-major from shared
//              memory, V MN-major), so S_{j+1} overlaps the softmax of S_j.
//   warps 2-5  softmax, one thread per query row (= TMEM lane): the row of S
//              in registers, causal / length mask on diagonal blocks, running
//              max and sum in fp32, P = exp2(S scale - m) rounded to bf16 into
//              swizzled shared memory. The running max is updated lazily: O
//              and the sum are rescaled only when the max grows by more than
//              2^8, so P stays <= 256 and the final O / l is unchanged (the
//              same max is used for the numerator and the denominator).
// At the end each thread reads its O row from TMEM, divides by its sum and
// writes bf16 to the shard's [token][h/N] output.
//
// Causal tiles stop at the diagonal block; heavy (late) query tiles launch
// first. Every barrier wait is bounded; a role that gives up records an error
// bit and the CTA leaves through the common exit after waiting (bounded) for
// its copies and MMAs in flight.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

constexpr int FA_BM = 128;                  // queries per CTA
constexpr int FA_BN = 128;                  // keys per block
constexpr int FA_D = 128;                   // head dim
constexpr int FA_THREADS = 192;
constexpr int FA_SUB = 128 * 128;           // one [128 rows][64 cols] bf16 box: 16 KB
constexpr int FA_TILE = 2 * FA_SUB;         // a [128][128] bf16 tile: 32 KB
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + FA_TILE;      // 2 buffers
constexpr int OFF_V = OFF_K + 2 * FA_TILE;  // 2 buffers
constexpr int OFF_P = OFF_V + 2 * FA_TILE;  // 2 buffers
constexpr int OFF_BAR = OFF_P + 2 * FA_TILE;
constexpr int FA_NUM_BARS = 16;
constexpr int FA_SMEM = 1024 + OFF_BAR + FA_NUM_BARS * 8 + 16;
static_assert(FA_SMEM <= 232448, "shared memory budget");

// barrier indices
constexpr int B_Q = 0, B_KFULL = 1, B_VFULL = 3, B_KVEMPTY = 5, B_SFULL = 7, B_SFREE = 9,
              B_PFULL = 11, B_PFREE = 13, B_ODONE = 15;

struct AttnParams {
  int seq, batch, hps, hs, causal, nq;
  long long M;  // tokens per shard
  float scale_log2;
  unsigned* err;
};

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
  if (p.causal && qt + 1 < nb) nb = qt + 1;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_KFULL + b), 1);
      mbar_init(bar(B_VFULL + b), 1);
      mbar_init(bar(B_KVEMPTY + b), 1);
      mbar_init(bar(B_SFULL + b), 1);
      mbar_init(bar(B_SFREE + b), 4);
      mbar_init(bar(B_PFULL + b), 4);
      mbar_init(bar(B_PFREE + b), 1);
    }
    mbar_init(bar(B_ODONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tm);
  if (warp == 1) tmem_alloc(smem_u32(tmem_holder), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;  // S_0: cols 0-127, S_1: 128-255, O: 256-383

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(bar(B_Q), FA_TILE);
      tma_load_3d(s0 + OFF_Q, &tm, bar(B_Q), head * FA_D, row_base + q0, g);
      tma_load_3d(s0 + OFF_Q + FA_SUB, &tm, bar(B_Q), head * FA_D + 64, row_base + q0, g);
      int j = 0;
      for (; j < nb; ++j) {
        const int b = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(bar(B_KVEMPTY + b), ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const int krow = row_base + j * FA_BN;
        const uint32_t kd = s0 + OFF_K + b * FA_TILE, vd = s0 + OFF_V + b * FA_TILE;
        mbar_arrive_expect_tx(bar(B_KFULL + b), FA_TILE);
        tma_load_3d(kd, &tm, bar(B_KFULL + b), p.hs + head * FA_D, krow, g);
        tma_load_3d(kd + FA_SUB, &tm, bar(B_KFULL + b), p.hs + head * FA_D + 64, krow, g);
        mbar_arrive_expect_tx(bar(B_VFULL + b), FA_TILE);
        tma_load_3d(vd, &tm, bar(B_VFULL + b), 2 * p.hs + head * FA_D, krow, g);
        tma_load_3d(vd + FA_SUB, &tm, bar(B_VFULL + b), 2 * p.hs + head * FA_D + 64, krow, g);
      }
      if (!ok) {
        atomicOr(p.err, ERR_WAIT_ATTN);
        *abort_flag = 1;
      }
      // every load issued must land before the CTA exits
      int never = 0;
      if (!mbar_wait(bar(B_Q), 0, &never)) atomicOr(p.err, ERR_WAIT_DRAIN);
      for (int jj = (j >= 2 ? j - 2 : 0); jj < j; ++jj) {
        const int b = jj & 1;
        const uint32_t ph = (jj >> 1) & 1;
        if (!mbar_wait(bar(B_KFULL + b), ph, &never)) atomicOr(p.err, ERR_WAIT_DRAIN);
        if (!mbar_wait(bar(B_VFULL + b), ph, &never)) atomicOr(p.err, ERR_WAIT_DRAIN);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16_f32(FA_BM, FA_BN);
      constexpr uint32_t idesc_o = umma_idesc_bf16_f32_bmn(FA_BM, FA_D);
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag);
      for (int j = 0; ok && j <= nb; ++j) {
        if (j < nb) {
          const int b = j & 1;
          const uint32_t ph = (j >> 1) & 1;
          if (!mbar_wait(bar(B_KFULL + b), ph, abort_flag) ||
              !mbar_wait(bar(B_SFREE + b), ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kb = s0 + OFF_K + b * FA_TILE;
#pragma unroll
          for (int kk = 0; kk < FA_D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * FA_SUB + (kk & 3) * 32;
            umma_bf16(tmem + b * FA_BN, umma_desc_sw128(s0 + OFF_Q + off),
                      umma_desc_sw128(kb + off), idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(B_SFULL + b));
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int b = jj & 1;
          const uint32_t ph = (jj >> 1) & 1;
          if (!mbar_wait(bar(B_PFULL + b), ph, abort_flag) ||
              !mbar_wait(bar(B_VFULL + b), ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t pb = s0 + OFF_P + b * FA_TILE;
          const uint32_t vb = s0 + OFF_V + b * FA_TILE;
#pragma unroll
          for (int kk = 0; kk < FA_BN / 16; ++kk) {
            umma_bf16(tmem + 2 * FA_BN, umma_desc_sw128(pb + (kk >> 2) * FA_SUB + (kk & 3) * 32),
                      umma_desc_sw128_mn(vb + kk * 2048, FA_SUB), idesc_o,
                      (jj > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(bar(B_PFREE + b));
          umma_commit(bar(B_KVEMPTY + b));
        }
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
  } else {
    // ------------------------------------------------------------ softmax
    const int q = warp & 3;
    const int r = q * 32 + lane;  // query row within the tile = TMEM lane
    const int t = q0 + r;         // query position within the sequence
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nb; ++j) {
      const int b = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      if (!mbar_wait(bar(B_SFULL + b), ph, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[FA_BN];
#pragma unroll
      for (int c = 0; c < FA_BN / 32; ++c)
        tmem_ld_32x32b_x32(tmem + lane_addr + b * FA_BN + c * 32,
                           *reinterpret_cast<uint32_t(*)[32]>(&s[c * 32]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_SFREE + b));

      const int k0 = j * FA_BN;
      if (k0 + FA_BN > p.seq || (p.causal && k0 + FA_BN - 1 > q0)) {
#pragma unroll
        for (int c = 0; c < FA_BN; ++c) {
          const int key = k0 + c;
          if (key >= p.seq || (p.causal && key > t)) s[c] = -INFINITY;
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < FA_BN; ++c) mx = fmaxf(mx, s[c]);
      // lazy max: move it (and rescale) only when exp2 would exceed 2^8
      const bool need = (mx != -INFINITY) && ((mx - m_used) * sl2 > 8.f);
      float alpha = 1.f;
      if (need) {
        alpha = exp2f((m_used - mx) * sl2);  // 0 when m_used is still -inf
        l *= alpha;
        m_used = mx;
      }
      if (__any_sync(0xffffffffu, need && j > 0)) {
        // O holds blocks < j: wait for PV_{j-1}, then O *= alpha on this row
        const int jp = j - 1;
        if (!mbar_wait(bar(B_PFREE + (jp & 1)), (jp >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < FA_D / 32; ++c) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(tmem + lane_addr + 2 * FA_BN + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st_32x32b_x32(tmem + lane_addr + 2 * FA_BN + c * 32, o);
        }
        tmem_st_wait();
      }
      const float base = (m_used == -INFINITY) ? 0.f : m_used * sl2;
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < FA_BN; ++c) {
        s[c] = exp2f(fmaf(s[c], sl2, -base));
        sum += s[c];
      }
      l += sum;
      // P_j -> shared buffer b once PV_{j-2} has read it
      if (!mbar_wait(bar(B_PFREE + b), ph ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t prow = s0 + OFF_P + b * FA_TILE + static_cast<uint32_t>(r) * 128u;
#pragma unroll
      for (int ch = 0; ch < FA_BN / 8; ++ch) {
        const uint32_t addr = prow + (ch >> 3) * FA_SUB +
                              ((static_cast<uint32_t>(ch & 7) ^ static_cast<uint32_t>(r & 7)) << 4);
        st_shared_v4(addr, pack_bf16x2(s[8 * ch + 0], s[8 * ch + 1]),
                     pack_bf16x2(s[8 * ch + 2], s[8 * ch + 3]),
                     pack_bf16x2(s[8 * ch + 4], s[8 * ch + 5]),
                     pack_bf16x2(s[8 * ch + 6], s[8 * ch + 7]));
      }
      fence_proxy_async_shared();
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
      uint16_t* orow = O + (static_cast<int64_t>(g) * p.M + row_base + t) * p.hs + head * FA_D;
#pragma unroll 1
      for (int c = 0; c < FA_D / 32; ++c) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tmem + lane_addr + 2 * FA_BN + c * 32, o);
        tmem_ld_wait();
        if (t < p.seq) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * e + 0]) * inv, __uint_as_float(o[8 * e + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + 8 * e) = v;
          }
        }
      }
    } else {
      if (lane == 0) atomicOr(p.err, ERR_WAIT_ATTN);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
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

int launch_attention(const void* QKV, int64_t batch, int64_t seq, int64_t h, int64_t n_heads,
                     int n_shards, int causal, void* O, cudaStream_t s, unsigned* err) {
  const int hps = static_cast<int>(n_heads / n_shards);
  const int64_t hs = h / n_shards;
  const int64_t M = batch * seq;
  auto enc = attn_map_encoder();
  if (enc == nullptr) return 1;
  CUtensorMap tm;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(3 * hs), static_cast<cuuint64_t>(M),
                        static_cast<cuuint64_t>(n_shards)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(3 * hs * 2),
                           static_cast<cuuint64_t>(M * 3 * hs * 2)};
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
  p.hs = static_cast<int>(hs);
  p.causal = causal;
  p.nq = static_cast<int>((seq + FA_BM - 1) / FA_BM);
  p.M = M;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(h / n_heads));
  p.err = err;
  cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, FA_SMEM);
  const dim3 grid(p.nq, static_cast<unsigned>(n_shards * batch * hps));
  attention_tc_kernel<<<grid, FA_THREADS, FA_SMEM, s>>>(tm, static_cast<uint16_t*>(O), p);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
