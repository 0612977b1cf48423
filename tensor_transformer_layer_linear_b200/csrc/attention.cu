// Local self-attention of every shard's heads on the 5th-generation tensor
// cores.
//
// "Tensor Parallelism in Large Language Models", "Local Self-Attention
// Computation": each GPU evaluates Head = softmax(Q K^T / sqrt(d_k)) V for
// its own heads with no communication. With the shards held on one GPU, one
// launch covers every (shard, sequence, local head, 128-query tile).
//
// One CTA per pair of 128-query tiles (256 queries, d = 128), 12 warps in
// three warpgroups:
//   WG0, WG1   softmax of query tile 0 / 1: one thread per query row (= TMEM
//              lane). The row of S is read from TMEM into registers once,
//              masked on diagonal / tail blocks, its max taken, P =
//              exp2(S scale - m) formed in fp32 with the row sum, and P stored
//              as bf16 pairs back into TMEM over the S columns. The running
//              max moves lazily: O and the sum are rescaled only when the max
//              grows by more than 2^8, so P stays <= 256 and O / l is
//              unchanged (the same max scales numerator and denominator).
//              These warpgroups raise their register limit with setmaxnreg.
//   WG2        warp 8: TMA (both Q tiles once, then 128-key K and V blocks
//              into 2-deep rings straight out of the QKV projection's
//              [shard][token][3h/N] output, 128-byte swizzle); warp 9: TMEM
//              owner and the single MMA-issuing thread; warps 10-11 idle.
//              WG2 lowers its register limit.
// MMA issue order per key block j (tiles 0, 1):
//   S_j^0 = Q_0 K_j^T | O_1 += P_{j-1}^1 V_{j-1} | S_j^1 = Q_1 K_j^T |
//   O_0 += P_j^0 V_j
// so each tile's softmax overlaps two MMAs of the other tile. S and P of a
// tile share TMEM columns: the S of the next block is issued right after the
// PV that reads P, relying on tcgen05.mma operations of one thread executing
// in issue order; a commit after S_j^T therefore also covers PV_{j-1}^T, which
// is what makes the softmax's O rescale safe without a further wait.
// TMEM: tile T uses columns [128 T, 128 T + 128) for S / P and
// [256 + 128 T, 384 + 128 T) for O.
// Causal CTAs stop at the diagonal block of their second tile; heavy (late)
// query tiles launch first. Every barrier wait is bounded; a role that gives
// up records an error bit and the CTA leaves through the common exit after
// waiting (bounded) for its copies and MMAs in flight.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

constexpr int FA_TILES = 2;                 // 128-query tiles per CTA
constexpr int FA_BM = 128;                  // queries per tile
constexpr int FA_BN = 128;                  // keys per block
constexpr int FA_D = 128;                   // head dim
constexpr int FA_THREADS = 384;             // 3 warpgroups
// Register split (setmaxnreg): the kernel is launched with 168 registers per
// thread (384 x 168 = 64512); the two softmax warpgroups rise to 208 and the
// load/MMA warpgroup drops to 72: 256 x 208 + 128 x 72 = 62464 <= 64512.
// The build checks the launch register count of this kernel.
constexpr int FA_REGS_LAUNCH = 168;
constexpr int FA_REGS_SOFTMAX = 208;
constexpr int FA_REGS_OTHER = 72;
static_assert(256 * FA_REGS_SOFTMAX + 128 * FA_REGS_OTHER <= FA_THREADS * FA_REGS_LAUNCH,
              "register split exceeds the launch allocation");
constexpr int FA_SUB = 128 * 128;           // one [128 rows][64 cols] bf16 box: 16 KB
constexpr int FA_TILE = 2 * FA_SUB;         // a [128][128] bf16 tile: 32 KB
constexpr int OFF_Q = 0;                    // FA_TILES tiles
constexpr int OFF_K = OFF_Q + FA_TILES * FA_TILE;  // 2 buffers
constexpr int OFF_V = OFF_K + 2 * FA_TILE;         // 2 buffers
constexpr int OFF_BAR = OFF_V + 2 * FA_TILE;
constexpr int FA_NUM_BARS = 16;
constexpr int FA_SMEM = 1024 + OFF_BAR + FA_NUM_BARS * 8 + 16;
static_assert(FA_SMEM <= 232448, "shared memory budget");

// barrier indices
constexpr int B_Q = 0, B_KFULL = 1, B_VFULL = 3, B_KEMPTY = 5, B_VEMPTY = 7, B_SFULL = 9,
              B_PFULL = 11, B_ODONE = 13;

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
  const int wg = warp >> 2;
  const int qt = p.causal ? (p.nq - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x);
  const int y = blockIdx.y;
  const int head = y % p.hps;
  const int sidx = (y / p.hps) % p.batch;
  const int g = y / (p.hps * p.batch);
  const int q0 = qt * FA_BM * FA_TILES;
  const int row_base = sidx * p.seq;  // first token of this sequence within the shard
  int nb = (p.seq + FA_BN - 1) / FA_BN;
  if (p.causal) {
    const int last = (q0 + FA_BM * FA_TILES - 1) / FA_BN + 1;
    if (last < nb) nb = last;
  }

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_KFULL + b), 1);
      mbar_init(bar(B_VFULL + b), 1);
      mbar_init(bar(B_KEMPTY + b), 1);
      mbar_init(bar(B_VEMPTY + b), 1);
      mbar_init(bar(B_SFULL + b), 1);   // per tile
      mbar_init(bar(B_PFULL + b), 4);   // per tile, one arrival per softmax warp
    }
    mbar_init(bar(B_ODONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8 && lane == 0) tma_prefetch_desc(&tm);
  if (warp == 9) tmem_alloc(smem_u32(tmem_holder), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (wg == 2) {
    setmaxnreg_dec<FA_REGS_OTHER>();
    if (warp == 8 && lane == 0) {
      // ---------------------------------------------------------- TMA
      bool ok = true;
      mbar_arrive_expect_tx(bar(B_Q), FA_TILES * FA_TILE);
      for (int T = 0; T < FA_TILES; ++T) {
        const int qrow = row_base + q0 + T * FA_BM;
        tma_load_3d(s0 + OFF_Q + T * FA_TILE, &tm, bar(B_Q), head * FA_D, qrow, g);
        tma_load_3d(s0 + OFF_Q + T * FA_TILE + FA_SUB, &tm, bar(B_Q), head * FA_D + 64, qrow, g);
      }
      const int kvh = head / p.group;  // this query head's local kv head
      const int kcol = p.q_w + kvh * FA_D, vcol = p.q_w + p.kv_w + kvh * FA_D;
      int kj = 0, vj = 0;  // K and V blocks issued
      for (int j = 0; j < nb; ++j) {
        const int b = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int krow = row_base + j * FA_BN;
        if (!mbar_wait(bar(B_KEMPTY + b), ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t kd = s0 + OFF_K + b * FA_TILE;
        mbar_arrive_expect_tx(bar(B_KFULL + b), FA_TILE);
        tma_load_3d(kd, &tm, bar(B_KFULL + b), kcol, krow, g);
        tma_load_3d(kd + FA_SUB, &tm, bar(B_KFULL + b), kcol + 64, krow, g);
        ++kj;
        if (!mbar_wait(bar(B_VEMPTY + b), ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t vd = s0 + OFF_V + b * FA_TILE;
        mbar_arrive_expect_tx(bar(B_VFULL + b), FA_TILE);
        tma_load_3d(vd, &tm, bar(B_VFULL + b), vcol, krow, g);
        tma_load_3d(vd + FA_SUB, &tm, bar(B_VFULL + b), vcol + 64, krow, g);
        ++vj;
      }
      if (!ok) {
        atomicOr(p.err, ERR_WAIT_ATTN);
        *abort_flag = 1;
      }
      // every load issued must land before the CTA exits
      int never = 0;
      if (!mbar_wait(bar(B_Q), 0, &never)) atomicOr(p.err, ERR_WAIT_DRAIN);
      for (int jj = (kj >= 2 ? kj - 2 : 0); jj < kj; ++jj)
        if (!mbar_wait(bar(B_KFULL + (jj & 1)), (jj >> 1) & 1, &never))
          atomicOr(p.err, ERR_WAIT_DRAIN);
      for (int jj = (vj >= 2 ? vj - 2 : 0); jj < vj; ++jj)
        if (!mbar_wait(bar(B_VFULL + (jj & 1)), (jj >> 1) & 1, &never))
          atomicOr(p.err, ERR_WAIT_DRAIN);
    } else if (warp == 9 && lane == 0) {
      // ---------------------------------------------------------- MMA
      constexpr uint32_t idesc_s = umma_idesc_bf16_f32(FA_BM, FA_BN);
      constexpr uint32_t idesc_o = umma_idesc_bf16_f32_bmn(FA_BM, FA_D);
      // descriptors built once; each MMA moves them by a constant offset
      // (the issuing thread shares its sub-partition with softmax warps, so
      // fewer instructions per MMA keep the tensor pipe fed)
      const uint64_t dq0 = umma_desc_sw128(s0 + OFF_Q), dq1 = umma_desc_sw128(s0 + OFF_Q + FA_TILE);
      const uint64_t dk0 = umma_desc_sw128(s0 + OFF_K), dk1 = umma_desc_sw128(s0 + OFF_K + FA_TILE);
      const uint64_t dv0 = umma_desc_sw128_mn(s0 + OFF_V, FA_SUB);
      const uint64_t dv1 = umma_desc_sw128_mn(s0 + OFF_V + FA_TILE, FA_SUB);
      auto qk = [&](int T, int b) {
        const uint64_t dq = T ? dq1 : dq0, dk = b ? dk1 : dk0;
#pragma unroll
        for (int kk = 0; kk < FA_D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * FA_SUB + (kk & 3) * 32;
          umma_bf16(tmem + T * FA_BN, desc_advance(dq, off), desc_advance(dk, off), idesc_s,
                    kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(B_SFULL + T));
      };
      auto pv = [&](int T, int b, bool first) {
        const uint64_t dv = b ? dv1 : dv0;
#pragma unroll
        for (int kk = 0; kk < FA_BN / 16; ++kk) {
          umma_bf16_tmem_a(tmem + 2 * FA_BN + T * FA_D, tmem + T * FA_BN + kk * 8,
                           desc_advance(dv, kk * 2048), idesc_o, (!first || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag);
      for (int j = 0; ok && j < nb; ++j) {
        const int b = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(bar(B_KFULL + b), ph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        qk(0, b);                                               // S_j^0
        if (j >= 1) {                                           // O_1 += P_{j-1}^1 V_{j-1}
          if (!mbar_wait(bar(B_PFULL + 1), (j - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          pv(1, (j - 1) & 1, j - 1 == 0);
          umma_commit(bar(B_VEMPTY + ((j - 1) & 1)));
        }
        qk(1, b);                                               // S_j^1
        umma_commit(bar(B_KEMPTY + b));
        if (!mbar_wait(bar(B_VFULL + b), ph, abort_flag) ||     // O_0 += P_j^0 V_j
            !mbar_wait(bar(B_PFULL + 0), j & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        pv(0, b, j == 0);
      }
      if (ok) {                                                 // O_1 += P_last^1 V_last
        const int jl = nb - 1;
        if (mbar_wait(bar(B_PFULL + 1), jl & 1, abort_flag)) {
          tc_fence_after();
          pv(1, jl & 1, jl == 0);
          umma_commit(bar(B_VEMPTY + (jl & 1)));
        } else {
          ok = false;
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
    setmaxnreg_inc<FA_REGS_SOFTMAX>();
    // ------------------------------------------------------------ softmax
    const int T = wg;               // query tile of this warpgroup
    const int q = warp & 3;         // TMEM lanes [32 q, 32 q + 32)
    const int r = q * 32 + lane;    // row within the tile
    const int t0 = q0 + T * FA_BM;  // first query of the tile
    const int t = t0 + r;           // query position within the sequence
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t s_cols = tmem + lane_addr + T * FA_BN;
    const uint32_t o_cols = tmem + lane_addr + 2 * FA_BN + T * FA_D;
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nb; ++j) {
      if (!mbar_wait(bar(B_SFULL + T), j & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int k0 = j * FA_BN;
      uint32_t v[FA_BN];
#pragma unroll
      for (int c = 0; c < FA_BN / 32; ++c) tmem_ld_32x32b_x32(s_cols + c * 32, &v[c * 32]);
      tmem_ld_wait();
      if (k0 + FA_BN > p.seq || (p.causal && k0 + FA_BN - 1 > t0)) {
#pragma unroll
        for (int e = 0; e < FA_BN; ++e) {
          const int key = k0 + e;
          if (key >= p.seq || (p.causal && key > t)) v[e] = 0xFF800000u;  // -inf
        }
      }
      float m8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) m8[e] = __uint_as_float(v[e]);
#pragma unroll
      for (int e = 8; e < FA_BN; ++e) m8[e & 7] = fmaxf(m8[e & 7], __uint_as_float(v[e]));
      const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      // lazy max: move it (and rescale) only when exp2 would exceed 2^8
      const bool need = (mx != -INFINITY) && ((mx - m_used) * sl2 > 8.f);
      float alpha = 1.f;
      if (need) {
        alpha = exp2f((m_used - mx) * sl2);  // 0 when m_used is still -inf
        l *= alpha;
        m_used = mx;
      }
      if (__any_sync(0xffffffffu, need && j > 0)) {
        // O holds blocks < j; PV_{j-1} of this tile completed before S_j
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
      if (lane == 0) mbar_arrive(bar(B_PFULL + T));
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
  if (warp == 9) {
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
  p.nq = static_cast<int>((seq + FA_BM * FA_TILES - 1) / (FA_BM * FA_TILES));
  p.M = M;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(FA_D));
  p.lse = lse;
  p.lse_stride = M + 128;
  p.err = err;
  // The setmaxnreg split assumes FA_REGS_LAUNCH registers per thread at
  // launch; with fewer, the softmax warpgroups' increase could never be
  // granted, so refuse to launch.
  static int launch_regs = -1;
  if (launch_regs < 0) {
    cudaFuncAttributes fa;
    launch_regs = cudaFuncGetAttributes(&fa, attention_tc_kernel) == cudaSuccess ? fa.numRegs : 0;
  }
  if (launch_regs * FA_THREADS < 256 * FA_REGS_SOFTMAX + 128 * FA_REGS_OTHER) return 3;
  cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, FA_SMEM);
  const dim3 grid(p.nq, static_cast<unsigned>(n_shards * batch * hps));
  attention_tc_kernel<<<grid, FA_THREADS, FA_SMEM, s>>>(tm, static_cast<uint16_t*>(O), p);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
