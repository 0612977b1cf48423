// Local self-attention of every shard's heads on the 5th-generation tensor
// cores.
//
// "Tensor Parallelism in Large Language Models", "Local Self-Attention
// Computation": each GPU evaluates Head = softmax(Q K^T / sqrt(d_k)) V for
// its own heads with no communication. With the shards held on one GPU, one
// launch covers every (shard, sequence, local head, 128-query tile).
//
// A persistent kernel: one CTA per SM, each walking a share of the 128-query
// tiles (d = 128), heaviest first; 8 warps:
//   warps 0-3  softmax: one thread per query row (= TMEM lane). The row of S
//              is read from TMEM into registers, masked on diagonal / tail
//              blocks, its max taken, P = exp2(S scale - m) formed in fp32
//              with the row sum, and P stored as bf16 pairs back into TMEM
//              over the S columns. The running max moves lazily: O and the
//              sum are rescaled only when the max grows by more than 2^8, so
//              P stays <= 256 and O / l is unchanged (the same max scales
//              numerator and denominator). A tile's O is normalised and
//              stored once the next tile's first P is formed, so the wait for
//              the tile's last PV overlaps that work.
//   warp 4     TMA: each tile's Q into a 2-deep ring (the next tile's Q loads
//              while the current one runs), then 128-key K blocks into a
//              2-deep ring straight out of the QKV projection's
//              [shard][token][3h/N] output (128-byte swizzle).
//   warp 6     TMA: the V blocks into their own 2-deep ring.
//   warp 5     TMEM owner and the single MMA-issuing thread.
// S has three buffers in TMEM, so the MMAs of the next key blocks overlap
// the softmax of the current one. Blocks are numbered over the CTA's whole
// work list, and the MMA order is
//   S_0 = Q K_0^T | S_1 | S_2 | O = P_0 V_0 | S_3 | O += P_1 V_1 | S_4 | ...
// running on across tile boundaries (S of the next tile's first blocks is
// computed while the softmax finishes the current tile). S_{n+3} overwrites
// the buffer holding P_n right after the MMA that reads it, relying on one
// thread's tcgen05.mma operations executing in issue order. A commit after
// every PV tells the softmax when O holds exactly the blocks before its own
// (needed only for a rescale); a commit after a tile's last PV releases its O
// to the softmax warps, whose next P arrival in turn releases the columns.
// When the softmax sees S_n, PV_{n-3} is complete but PV_{n-2} may not be,
// so both commits alternate between two barriers (by block and by tile
// parity): a parity wait on one barrier is then never two phases behind.
// TMEM: S / P buffer b at columns [128 b, 128 b + 128) (b < 3), O at
// [384, 512).
// Causal tiles stop at their diagonal block. Every barrier wait is bounded;
// a role that gives up records an error bit and the CTA leaves through the
// common exit after waiting (bounded) for its copies and MMAs in flight.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

constexpr int FA_BM = 128;                  // queries per tile
constexpr int FA_BN = 128;                  // keys per block
constexpr int FA_D = 128;                   // head dim
constexpr int FA_THREADS = 256;             // 8 warps: up to 255 registers per thread
constexpr int FA_SUB = 128 * 128;           // one [128 rows][64 cols] bf16 box: 16 KB
constexpr int FA_TILE = 2 * FA_SUB;         // a [128][128] bf16 tile: 32 KB
constexpr int OFF_Q = 0;                    // 2 buffers (the next tile's Q loads early)
constexpr int OFF_K = OFF_Q + 2 * FA_TILE;  // 2 buffers
constexpr int OFF_V = OFF_K + 2 * FA_TILE;  // 2 buffers
constexpr int OFF_BAR = OFF_V + 2 * FA_TILE;
constexpr int FA_NUM_BARS = 23;
constexpr int FA_SBUF = 3;                  // S / P buffers in TMEM
constexpr int FA_SMEM = 1024 + OFF_BAR + FA_NUM_BARS * 8 + 16;
static_assert(FA_SMEM <= 232448, "shared memory budget");

// barrier indices (Q, K, V, S and P per buffer b)
constexpr int B_QFULL = 0, B_QEMPTY = 2, B_KFULL = 4, B_KEMPTY = 6, B_VFULL = 8, B_VEMPTY = 10,
              B_SFULL = 12, B_PFULL = 15, B_OUPD = 18, B_ODONE = 20, B_DRAIN = 22;

struct AttnParams {
  int seq, batch, hps, causal, nq;
  int n_units;  // (shard, sequence, local head) triples
  int q_w;    // query columns per shard (query heads per shard x 128)
  int kv_w;   // key (= value) columns per shard
  int group;  // local query heads per local kv head
  long long M;  // tokens per shard
  float scale_log2;
  float* lse;  // optional: base-2 log-sum-exp of each query's scaled scores
  long long lse_stride;  // per (shard, head): tokens per shard + 128
  unsigned* err;
};

// One query tile of the work list. Tiles are ordered heaviest first (for
// causal attention, the latest query tiles see the most key blocks) and dealt
// to the persistent CTAs in a snake: CTA c takes tile k G + c in even rounds k
// and k G + G - 1 - c in odd ones (G CTAs), which evens out the causal work.
struct AttnTile {
  bool valid;
  int head, g, q0, row_base, nb, kcol, vcol;
};

__device__ __forceinline__ AttnTile attn_tile(const AttnParams& p, int round) {
  AttnTile t;
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const int w = round * G + ((round & 1) ? (G - 1 - c) : c);
  t.valid = w < p.nq * p.n_units;
  const int wi = t.valid ? w : 0;
  const int qi = wi / p.n_units, y = wi % p.n_units;
  const int qt = p.causal ? (p.nq - 1 - qi) : qi;
  t.head = y % p.hps;
  const int sidx = (y / p.hps) % p.batch;
  t.g = y / (p.hps * p.batch);
  t.q0 = qt * FA_BM;
  t.row_base = sidx * p.seq;  // first token of the sequence within the shard
  t.nb = (p.seq + FA_BN - 1) / FA_BN;
  if (p.causal) {
    const int last = (t.q0 + FA_BM - 1) / FA_BN + 1;
    if (last < t.nb) t.nb = last;
  }
  const int kvh = t.head / p.group;  // the query head's local kv head
  t.kcol = p.q_w + kvh * FA_D;
  t.vcol = p.q_w + p.kv_w + kvh * FA_D;
  return t;
}

// Packed two-wide fp32 FMA and add (sm_100: one instruction for two values):
// the softmax forms S scale - m and accumulates the row sum a pair at a time,
// half the FMA-pipe instructions of the scalar forms.
__device__ __forceinline__ uint64_t pack_f32x2(uint32_t lo, uint32_t hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
  return d;
}
__device__ __forceinline__ void unpack_f32x2(uint64_t v, float& lo, float& hi) {
  uint32_t a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(v));
  lo = __uint_as_float(a);
  hi = __uint_as_float(b);
}
__device__ __forceinline__ uint64_t ffma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

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

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_QFULL + b), 1);
      mbar_init(bar(B_QEMPTY + b), 1);
      mbar_init(bar(B_KFULL + b), 1);
      mbar_init(bar(B_KEMPTY + b), 1);
      mbar_init(bar(B_VFULL + b), 1);
      mbar_init(bar(B_VEMPTY + b), 1);
    }
    for (int b = 0; b < FA_SBUF; ++b) {
      mbar_init(bar(B_SFULL + b), 1);
      mbar_init(bar(B_PFULL + b), 4);  // one arrival per softmax warp
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_OUPD + b), 1);   // PV of blocks b, b + 2, ... complete
      mbar_init(bar(B_ODONE + b), 1);  // O of tiles b, b + 2, ... complete
    }
    mbar_init(bar(B_DRAIN), 1);
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
    // Blocks are counted over the CTA's whole work list, so the rings run on
    // across tile boundaries and the next tile's Q and first K / V blocks
    // load while the current tile finishes.
    if (lane == 0) {
      const bool is_k = warp == 4;
      const int full = is_k ? B_KFULL : B_VFULL, empty = is_k ? B_KEMPTY : B_VEMPTY;
      const uint32_t ring = s0 + (is_k ? OFF_K : OFF_V);
      bool ok = true;
      int nblk = 0, ntile = 0;  // blocks and tiles issued
      for (int round = 0; ok; ++round) {
        const AttnTile t = attn_tile(p, round);
        if (!t.valid) break;
        if (is_k) {
          const int qb = ntile & 1;
          if (!mbar_wait(bar(B_QEMPTY + qb), ((ntile >> 1) & 1) ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(B_QFULL + qb), FA_TILE);
          const uint32_t qd = s0 + OFF_Q + qb * FA_TILE;
          tma_load_3d(qd, &tm, bar(B_QFULL + qb), t.head * FA_D, t.row_base + t.q0, t.g);
          tma_load_3d(qd + FA_SUB, &tm, bar(B_QFULL + qb), t.head * FA_D + 64, t.row_base + t.q0,
                      t.g);
        }
        ++ntile;
        const int col = is_k ? t.kcol : t.vcol;
        for (int j = 0; j < t.nb; ++j) {
          const int b = nblk & 1;
          if (!mbar_wait(bar(empty + b), ((nblk >> 1) & 1) ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t d = ring + b * FA_TILE;
          const int krow = t.row_base + j * FA_BN;
          mbar_arrive_expect_tx(bar(full + b), FA_TILE);
          tma_load_3d(d, &tm, bar(full + b), col, krow, t.g);
          tma_load_3d(d + FA_SUB, &tm, bar(full + b), col + 64, krow, t.g);
          ++nblk;
        }
      }
      if (!ok) {
        atomicOr(p.err, ERR_WAIT_ATTN);
        *abort_flag = 1;
      }
      // every load issued must land before the CTA exits
      int never = 0;
      if (is_k)
        for (int i = (ntile >= 2 ? ntile - 2 : 0); i < ntile; ++i)
          if (!mbar_wait(bar(B_QFULL + (i & 1)), (i >> 1) & 1, &never))
            atomicOr(p.err, ERR_WAIT_DRAIN);
      for (int jj = (nblk >= 2 ? nblk - 2 : 0); jj < nblk; ++jj)
        if (!mbar_wait(bar(full + (jj & 1)), (jj >> 1) & 1, &never))
          atomicOr(p.err, ERR_WAIT_DRAIN);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA
    // Two cursors walk the work list: the QK^T cursor runs two blocks ahead
    // of the PV cursor (S is double-buffered), across tile boundaries.
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16_f32(FA_BM, FA_BN);
      constexpr uint32_t idesc_o = umma_idesc_bf16_f32_bmn(FA_BM, FA_D);
      // descriptors built once; each MMA moves them by a constant offset
      const uint64_t dq0 = umma_desc_sw128(s0 + OFF_Q), dq1 = umma_desc_sw128(s0 + OFF_Q + FA_TILE);
      const uint64_t dk0 = umma_desc_sw128(s0 + OFF_K), dk1 = umma_desc_sw128(s0 + OFF_K + FA_TILE);
      const uint64_t dv0 = umma_desc_sw128_mn(s0 + OFF_V, FA_SUB);
      const uint64_t dv1 = umma_desc_sw128_mn(s0 + OFF_V + FA_TILE, FA_SUB);
      struct Cursor {
        AttnTile t;
        int round, tile, j, blk;  // work-list round, local tile, block within it, global block
      };
      Cursor cq{attn_tile(p, 0), 0, 0, 0, 0};
      Cursor cp = cq;
      auto advance = [&](Cursor& c) {
        ++c.blk;
        if (++c.j == c.t.nb) {
          c.j = 0;
          ++c.tile;
          c.t = attn_tile(p, ++c.round);
        }
      };
      bool ok = true;
      // S_blk = Q K_blk^T into buffer blk % FA_SBUF (K from ring slot blk & 1)
      auto qk = [&]() -> bool {
        const int qb = cq.tile & 1, b = cq.blk & 1, sb = cq.blk % FA_SBUF;
        if (cq.j == 0 && !mbar_wait(bar(B_QFULL + qb), (cq.tile >> 1) & 1, abort_flag)) return false;
        if (!mbar_wait(bar(B_KFULL + b), (cq.blk >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dq = qb ? dq1 : dq0, dk = b ? dk1 : dk0;
#pragma unroll
        for (int kk = 0; kk < FA_D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * FA_SUB + (kk & 3) * 32;
          umma_bf16(tmem + sb * FA_BN, desc_advance(dq, off), desc_advance(dk, off), idesc_s,
                    kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(B_KEMPTY + b));
        umma_commit(bar(B_SFULL + sb));
        if (cq.j == cq.t.nb - 1) umma_commit(bar(B_QEMPTY + qb));  // the tile's last QK^T
        advance(cq);
        return true;
      };
      for (int n = 0; ok && n < FA_SBUF && cq.t.valid; ++n) ok = qk();
      while (ok && cp.t.valid) {
        const int b = cp.blk & 1, pb = cp.blk % FA_SBUF;
        const uint32_t ph = (cp.blk >> 1) & 1, pph = (cp.blk / FA_SBUF) & 1;
        if (!mbar_wait(bar(B_VFULL + b), ph, abort_flag) ||
            !mbar_wait(bar(B_PFULL + pb), pph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t dv = b ? dv1 : dv0;
#pragma unroll
        for (int kk = 0; kk < FA_BN / 16; ++kk)             // O (+)= P V
          umma_bf16_tmem_a(tmem + FA_SBUF * FA_BN, tmem + pb * FA_BN + kk * 8,
                           desc_advance(dv, kk * 2048), idesc_o, (cp.j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(B_VEMPTY + b));
        umma_commit(bar(B_OUPD + (cp.blk & 1)));
        if (cp.j == cp.t.nb - 1) umma_commit(bar(B_ODONE + (cp.tile & 1)));  // the tile's O is complete
        advance(cp);
        if (cq.t.valid) ok = qk();                           // reuses the buffer P was in
      }
      if (!ok) {
        atomicOr(p.err, ERR_WAIT_ATTN);
        *abort_flag = 1;
      }
      // drain every MMA this thread issued
      umma_commit(bar(B_DRAIN));
      int never = 0;
      if (!mbar_wait(bar(B_DRAIN), 0, &never)) atomicOr(p.err, ERR_WAIT_DRAIN);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ softmax
    const int r = warp * 32 + lane;  // row within the tile (= TMEM lane)
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t o_cols = tmem + lane_addr + FA_SBUF * FA_BN;
    const float sl2 = p.scale_log2;
    bool ok = true;
    // A tile's O: normalise and store it. It runs after the next tile's first
    // P is formed (its wait for the last PV overlaps that work) and before
    // that P's arrival, which is what lets the next tile's first PV
    // overwrite the O columns.
    auto epilogue = [&](const AttnTile& tl, int tile, float m_used, float l) -> bool {
      if (!mbar_wait(bar(B_ODONE + (tile & 1)), (tile >> 1) & 1, abort_flag)) return false;
      tc_fence_after();
      const int t = tl.q0 + r;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float base_final = (m_used == -INFINITY) ? 0.f : m_used * sl2;
      uint16_t* orow =
          O + (static_cast<int64_t>(tl.g) * p.M + tl.row_base + t) * p.q_w + tl.head * FA_D;
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
        p.lse[(static_cast<int64_t>(tl.g) * p.hps + tl.head) * p.lse_stride + tl.row_base + t] =
            base_final + log2f(l);
      return true;
    };
    AttnTile prev{};
    float prev_m = -INFINITY, prev_l = 0.f;
    bool pending = false;  // prev's O still to be stored
    int blk = 0;  // global block count of this CTA
    int tile = 0;
    for (int round = 0; ok; ++round, ++tile) {
      const AttnTile tl = attn_tile(p, round);
      if (!tl.valid) break;
      const int q0 = tl.q0;
      const int t = q0 + r;  // query position within the sequence
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < tl.nb; ++j, ++blk) {
        const int b = blk % FA_SBUF;
        if (!mbar_wait(bar(B_SFULL + b), (blk / FA_SBUF) & 1, abort_flag)) {
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
          // O must hold exactly the tile's blocks before j: wait for the previous PV
          if (!mbar_wait(bar(B_OUPD + ((blk - 1) & 1)), ((blk - 1) >> 1) & 1, abort_flag)) {
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
        const uint64_t sl2x2 = pack_f32x2(__float_as_uint(sl2), __float_as_uint(sl2));
        const uint64_t nbx2 = pack_f32x2(__float_as_uint(-base), __float_as_uint(-base));
        uint64_t s4[4] = {0ull, 0ull, 0ull, 0ull};  // row-sum pairs (+0.0f, +0.0f)
#pragma unroll
        for (int c = 0; c < FA_BN / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float xa, xb;
            unpack_f32x2(ffma_f32x2(pack_f32x2(v[c * 32 + e], v[c * 32 + e + 1]), sl2x2, nbx2), xa, xb);
            const float a = ex2_approx(xa);
            const float bb = ex2_approx(xb);
            s4[(e >> 1) & 3] = fadd_f32x2(s4[(e >> 1) & 3], pack_f32x2(__float_as_uint(a), __float_as_uint(bb)));
            pk[e >> 1] = pack_bf16x2(a, bb);
          }
          tmem_st_32x32b_x16(s_cols + c * 16, pk);
        }
        float s8[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) unpack_f32x2(s4[u], s8[2 * u], s8[2 * u + 1]);
        l += ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
        if (j == 0 && pending) {
          if (!epilogue(prev, tile - 1, prev_m, prev_l)) {
            ok = false;
            break;
          }
          pending = false;
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PFULL + b));
      }
      if (!ok) break;
      prev = tl;
      prev_m = m_used;
      prev_l = l;
      pending = true;
    }
    if (ok && pending && !epilogue(prev, tile - 1, prev_m, prev_l)) ok = false;
    if (!ok) {
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
                     int num_sms, float* lse) {
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
  p.n_units = static_cast<int>(n_shards * batch * hps);
  cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, FA_SMEM);
  // persistent: one CTA per SM (shared memory and TMEM admit one), each
  // walking its share of the query tiles
  if (num_sms <= 0) return 2;
  const int64_t tiles = static_cast<int64_t>(p.nq) * p.n_units;
  const dim3 grid(static_cast<unsigned>(tiles < num_sms ? tiles : num_sms));
  attention_tc_kernel<<<grid, FA_THREADS, FA_SMEM, s>>>(tm, static_cast<uint16_t*>(O), p);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
