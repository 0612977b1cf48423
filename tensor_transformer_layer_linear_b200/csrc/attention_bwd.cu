// Backward of the local self-attention of every shard's heads on the
// 5th-generation tensor cores.
//
// "Tensor Parallelism in Large Language Models", "Local Self-Attention
// Computation": the attention of a shard's heads is local, so its backward is
// local too; the block's single backward reduction comes after the QKV
// projection's input gradient (tp_attn_backward). With O = P V,
// P = softmax(S), S = Q K^T / sqrt(d):
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  D = rowsum(dO * O),
//   dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d),
// where P is rebuilt from the forward's log-sum-exp.
//
// One CTA per (shard, sequence, key/value head, 128-key block), 22 warps,
// stepping through the 64-query blocks of every query head that uses the
// key/value head (one for multi-head attention, the group for grouped-query
// attention: the key block's dK and dV sum over the group):
//   warp 0     TMA: the key block's K and V once, then each query block's Q
//              and dO into a 4-deep ring (128-byte swizzle), straight out of
//              the QKV projection's [shard][token][3h/N] output and dO, and
//              its lse and D into a 2-deep shared ring (bulk copies when the
//              rows are 16-byte aligned);
//   warp 1     TMEM owner and the single MMA-issuing thread;
//   warps 2-5  one thread per head-dimension column (TMEM lane): drain the
//              block's dQ^T from TMEM into an fp32 accumulator in global
//              memory with reductions (every key block of the sequence
//              contributes to it);
//   warps 6-21 four threads per key (TMEM lane), each for 16 of the block's
//              64 queries: P^T = exp2(S^T scale - lse), masked, stored as
//              bf16 pairs over the first 8 of the 16 S^T columns the thread
//              has read (the A operand of dV += P^T dO), and
//              dS^T = P^T * (dP^T - D) in bf16 into a swizzled shared tile,
//              the K-major A operand of dK += dS^T Q and the MN-major B
//              operand of dQ^T = K^T dS^T; at the end each writes 32 columns
//              of dK (scaled) and dV in bf16 through tiles in the (then idle)
//              Q ring and TMA tensor stores (direct stores for rows past the
//              sequence).
// S^T and dP^T are double-buffered in TMEM, so the tensor cores compute the
// next block's S^T = K Q^T and dP^T = V dO^T while the key threads work on
// the current one; dQ^T of a block lands in that block's dP^T columns once
// they are read. TMEM: buffer b in [128 b, 128 b + 128) (S^T, then P^T of
// queries [16 k, 16 k + 16) in its columns [16 k, 16 k + 8); dP^T, then dQ^T,
// in its last 64), dV
// [256, 384), dK [384, 512). Causal key blocks start at the first query block that sees
// them; the heaviest (first) key blocks launch first. Every barrier wait is
// bounded; a role that gives up records an error bit and the CTA leaves
// through the common exit after waiting (bounded) for its copies and MMAs in
// flight.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

constexpr int AB_BK = 128;        // keys per CTA
constexpr int AB_BQ = 64;         // queries per step
constexpr int AB_D = 128;         // head dim
constexpr int AB_THREADS = 704;  // 22 warps
constexpr int AB_NST = 4;         // Q / dO ring depth
constexpr int AB_KSUB = 128 * 128;          // [128 rows][64 cols] bf16: 16 KB
constexpr int AB_KTILE = 2 * AB_KSUB;       // [128][128] bf16: K or V
constexpr int AB_QSUB = 64 * 128;           // [64 rows][64 cols] bf16: 8 KB
constexpr int AB_QTILE = 2 * AB_QSUB;       // [64][128] bf16: Q or dO block
constexpr int AB_DSTILE = 128 * 128;        // dS^T [128 keys][64 queries] bf16: 16 KB
constexpr int AOFF_K = 0;
constexpr int AOFF_V = AOFF_K + AB_KTILE;
constexpr int AOFF_Q = AOFF_V + AB_KTILE;              // AB_NST stages
constexpr int AOFF_DO = AOFF_Q + AB_NST * AB_QTILE;    // AB_NST stages
constexpr int AOFF_DS = AOFF_DO + AB_NST * AB_QTILE;   // 2 buffers
constexpr int AOFF_LD = AOFF_DS + 2 * AB_DSTILE;       // 2 x (lse[64], D[64])
constexpr int AOFF_BAR = AOFF_LD + 2 * 2 * AB_BQ * 4;
constexpr int AB_NUM_BARS = 24;
constexpr int AB_SMEM = 1024 + AOFF_BAR + AB_NUM_BARS * 8 + 16;
static_assert(AB_SMEM <= 232448, "shared memory budget");

// barriers
constexpr int AB_KV = 0, AB_QFULL = 1, AB_QEMPTY = AB_QFULL + AB_NST,
              AB_SDP = AB_QEMPTY + AB_NST,     // 2: S^T and dP^T of buffer b computed
              AB_DS = AB_SDP + 2,              // 2: key threads done with buffer b
              AB_DQFULL = AB_DS + 2,           // 2: dQ^T in buffer b (and dK, dV done)
              AB_DQEMPTY = AB_DQFULL + 2,      // 2: dQ^T of buffer b drained
              AB_LDFULL = AB_DQEMPTY + 2,      // 2: lse / D stage loaded
              AB_LDEMPTY = AB_LDFULL + 2,      // 2: lse / D stage read
              AB_DONE = AB_LDEMPTY + 2;
static_assert(AB_DONE < AB_NUM_BARS, "barrier count");

struct AttnBwdParams {
  int seq, batch, hps, causal, nq;
  int kvl;       // key/value heads per shard
  int group;     // local query heads per local key/value head
  int q_w;       // query columns per shard (hps x 128)
  int ld;        // QKV row width per shard: q_w + 2 kvl x 128
  long long M;   // tokens per shard
  long long stride;  // M + 128: per-head row length of lse, D and dq_acc
  float scale_log2, scale;
  int ld_bulk;        // lse / D rows 16-byte aligned: copied by the TMA warp
  const float* lse;   // [N * hps][stride], base 2, by token
  const float* dsum;  // D, same layout
  float* dq_acc;      // [N * hps][stride][128] fp32
  uint16_t* dqkv;     // [N][M][3 hs]
  unsigned* err;
};

__device__ __forceinline__ void red_add_f32(float* addr, uint32_t v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(__uint_as_float(v)) : "memory");
}

__global__ void __launch_bounds__(AB_THREADS, 1)
    attention_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_kv,
                            const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_do,
                            const __grid_constant__ CUtensorMap tm_st, const AttnBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* sm = smem_raw + pad;
  const uint32_t s0 = smem_u32(sm);
  const uint32_t bar0 = s0 + AOFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + AOFF_BAR + AB_NUM_BARS * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int y = blockIdx.x;
  const int kvh = y % p.kvl;  // local key/value head
  const int sidx = (y / p.kvl) % p.batch;
  const int g = y / (p.kvl * p.batch);
  const int j = blockIdx.y;  // key block
  const int kv0 = j * AB_BK;
  const int row_base = sidx * p.seq;
  // first query block that sees a key of this block (causal: queries >= kv0)
  const int i_first = p.causal ? kv0 / AB_BQ : 0;
  const int n_qb = p.nq - i_first;  // query blocks per query head
  const int n_it = p.group * n_qb;  // (query head of the group, query block) steps
  // step t: query head kvh * group + t / n_qb (local), query block i_first + t % n_qb
  auto step_head = [&](int t) { return kvh * p.group + t / n_qb; };
  auto step_block = [&](int t) { return i_first + t % n_qb; };
  auto head_row = [&](int t) {  // (shard, query head) row of lse, D and dq_acc
    return static_cast<int64_t>(g) * p.hps + step_head(t);
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(AB_KV), 1);
    for (int s = 0; s < AB_NST; ++s) {
      mbar_init(bar(AB_QFULL + s), 1);
      mbar_init(bar(AB_QEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(AB_SDP + b), 1);
      mbar_init(bar(AB_DS + b), 16);      // one arrival per key warp
      mbar_init(bar(AB_DQFULL + b), 1);
      mbar_init(bar(AB_DQEMPTY + b), 4);  // one arrival per drain warp
      mbar_init(bar(AB_LDFULL + b), 1);
      mbar_init(bar(AB_LDEMPTY + b), 16); // one arrival per key warp
    }
    mbar_init(bar(AB_DONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_kv);
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_st);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_holder), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA
    bool ok = true;
    const int kcol = p.q_w + kvh * AB_D, vcol = p.q_w + p.kvl * AB_D + kvh * AB_D;
    mbar_arrive_expect_tx(bar(AB_KV), 2 * AB_KTILE);
    tma_load_3d(s0 + AOFF_K, &tm_kv, bar(AB_KV), kcol, row_base + kv0, g);
    tma_load_3d(s0 + AOFF_K + AB_KSUB, &tm_kv, bar(AB_KV), kcol + 64, row_base + kv0, g);
    tma_load_3d(s0 + AOFF_V, &tm_kv, bar(AB_KV), vcol, row_base + kv0, g);
    tma_load_3d(s0 + AOFF_V + AB_KSUB, &tm_kv, bar(AB_KV), vcol + 64, row_base + kv0, g);
    int issued = 0, ld_issued = 0;
    for (int it = 0; it < n_it; ++it) {
      const int st = it % AB_NST;
      const uint32_t ph = (it / AB_NST) & 1;
      if (!mbar_wait(bar(AB_QEMPTY + st), ph ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      const int q0 = step_block(it) * AB_BQ;
      const int qrow = row_base + q0;
      const int qcol = step_head(it) * AB_D;
      const uint32_t qd = s0 + AOFF_Q + st * AB_QTILE, dd = s0 + AOFF_DO + st * AB_QTILE;
      mbar_arrive_expect_tx(bar(AB_QFULL + st), 2 * AB_QTILE);
      tma_load_3d(qd, &tm_q, bar(AB_QFULL + st), qcol, qrow, g);
      tma_load_3d(qd + AB_QSUB, &tm_q, bar(AB_QFULL + st), qcol + 64, qrow, g);
      tma_load_3d(dd, &tm_do, bar(AB_QFULL + st), qcol, qrow, g);
      tma_load_3d(dd + AB_QSUB, &tm_do, bar(AB_QFULL + st), qcol + 64, qrow, g);
      ++issued;
      if (p.ld_bulk) {
        const int ls = it & 1;
        if (!mbar_wait(bar(AB_LDEMPTY + ls), ((it >> 1) & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t ld = s0 + AOFF_LD + ls * (2 * AB_BQ * 4);
        const int64_t lrow = head_row(it) * p.stride + row_base + q0;
        mbar_arrive_expect_tx(bar(AB_LDFULL + ls), 2 * AB_BQ * 4);
        bulk_load(ld, p.lse + lrow, AB_BQ * 4, bar(AB_LDFULL + ls));
        bulk_load(ld + AB_BQ * 4, p.dsum + lrow, AB_BQ * 4, bar(AB_LDFULL + ls));
        ++ld_issued;
      }
    }
    if (!ok) {
      atomicOr(p.err, ERR_WAIT_ATTN);
      *abort_flag = 1;
    }
    // every load issued must land before the CTA exits
    int never = 0;
    if (!mbar_wait(bar(AB_KV), 0, &never)) atomicOr(p.err, ERR_WAIT_DRAIN);
    for (int ii = (issued >= AB_NST ? issued - AB_NST : 0); ii < issued; ++ii)
      if (!mbar_wait(bar(AB_QFULL + ii % AB_NST), (ii / AB_NST) & 1, &never))
        atomicOr(p.err, ERR_WAIT_DRAIN);
    for (int ii = (ld_issued >= 2 ? ld_issued - 2 : 0); ii < ld_issued; ++ii)
      if (!mbar_wait(bar(AB_LDFULL + (ii & 1)), (ii >> 1) & 1, &never))
        atomicOr(p.err, ERR_WAIT_DRAIN);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA
    constexpr uint32_t idesc_s = umma_idesc_bf16_f32(AB_BK, AB_BQ);          // A, B K-major
    constexpr uint32_t idesc_kmn = umma_idesc_bf16_f32_bmn(AB_BK, AB_D);     // B MN-major
    constexpr uint32_t idesc_dq =
        umma_idesc_bf16_f32_bmn(AB_D, AB_BQ) | (1u << 15);                   // A, B MN-major
    const uint32_t sK = s0 + AOFF_K, sV = s0 + AOFF_V;
    // descriptors built once; each MMA moves them by a constant offset
    const uint64_t dK = umma_desc_sw128(sK), dV = umma_desc_sw128(sV);
    const uint64_t dK_mn = umma_desc_sw128_mn(sK, AB_KSUB);
    // S^T and dP^T of query block k into buffer k & 1
    auto issue_sdp = [&](int k) -> bool {
      const int st = k % AB_NST, b = k & 1;
      if (!mbar_wait(bar(AB_QFULL + st), (k / AB_NST) & 1, abort_flag)) return false;
      // the buffer's dQ^T of block k - 2 must be drained (its S^T / P^T and
      // dP^T were consumed before that dQ^T was computed)
      if (k >= 2 && !mbar_wait(bar(AB_DQEMPTY + b), ((k - 2) >> 1) & 1, abort_flag)) return false;
      tc_fence_after();
      const uint64_t dQ = umma_desc_sw128(s0 + AOFF_Q + st * AB_QTILE);
      const uint64_t dO = umma_desc_sw128(s0 + AOFF_DO + st * AB_QTILE);
      const uint32_t tS = tmem + 128u * b, tP = tS + 64u;
#pragma unroll
      for (int kk = 0; kk < AB_D / 16; ++kk) {   // contraction over d
        const uint32_t ka = (kk >> 2) * AB_KSUB + (kk & 3) * 32;
        const uint32_t qa = (kk >> 2) * AB_QSUB + (kk & 3) * 32;
        umma_bf16(tS, desc_advance(dK, ka), desc_advance(dQ, qa), idesc_s, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < AB_D / 16; ++kk) {
        const uint32_t ka = (kk >> 2) * AB_KSUB + (kk & 3) * 32;
        const uint32_t qa = (kk >> 2) * AB_QSUB + (kk & 3) * 32;
        umma_bf16(tP, desc_advance(dV, ka), desc_advance(dO, qa), idesc_s, kk > 0 ? 1u : 0u);
      }
      umma_commit(bar(AB_SDP + b));
      return true;
    };
    bool ok = mbar_wait(bar(AB_KV), 0, abort_flag);
    if (ok && n_it > 0) ok = issue_sdp(0);
    for (int it = 0; ok && it < n_it; ++it) {
      const int st = it % AB_NST, b = it & 1;
      if (it + 1 < n_it && !issue_sdp(it + 1)) {
        ok = false;
        break;
      }
      if (!mbar_wait(bar(AB_DS + b), (it >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t dQ_mn = umma_desc_sw128_mn(s0 + AOFF_Q + st * AB_QTILE, AB_QSUB);
      const uint64_t dO_mn = umma_desc_sw128_mn(s0 + AOFF_DO + st * AB_QTILE, AB_QSUB);
      const uint64_t dS_k = umma_desc_sw128(s0 + AOFF_DS + b * AB_DSTILE);
      const uint64_t dS_mn = umma_desc_sw128_mn(s0 + AOFF_DS + b * AB_DSTILE, AB_QSUB);
      const uint32_t tS = tmem + 128u * b, tP = tS + 64u;
      // dV += P^T dO: P^T (keys x queries, bf16 pairs) from TMEM
#pragma unroll
      for (int kk = 0; kk < AB_BQ / 16; ++kk)
        umma_bf16_tmem_a(tmem + 256u, tS + kk * 16,  // P^T of queries 16 kk.. (8 columns)
                         desc_advance(dO_mn, kk * 2048),
                         idesc_kmn, (it > 0 || kk > 0) ? 1u : 0u);
      // dK += dS^T Q
#pragma unroll
      for (int kk = 0; kk < AB_BQ / 16; ++kk)
        umma_bf16(tmem + 384u, desc_advance(dS_k, kk * 32), desc_advance(dQ_mn, kk * 2048),
                  idesc_kmn,
                  (it > 0 || kk > 0) ? 1u : 0u);
      // dQ^T = K^T dS^T (head dim x queries), contraction over the keys
#pragma unroll
      for (int kk = 0; kk < AB_BK / 16; ++kk)
        umma_bf16(tP, desc_advance(dK_mn, kk * 2048), desc_advance(dS_mn, kk * 2048), idesc_dq,
                  kk > 0 ? 1u : 0u);
      umma_commit(bar(AB_DQFULL + b));
      umma_commit(bar(AB_QEMPTY + st));
    }
    if (!ok) {
      atomicOr(p.err, ERR_WAIT_ATTN);
      *abort_flag = 1;
    }
    // done doubles as the drain of every MMA this thread issued
    umma_commit(bar(AB_DONE));
    int never = 0;
    if (!mbar_wait(bar(AB_DONE), 0, &never)) atomicOr(p.err, ERR_WAIT_DRAIN);
  } else if (warp >= 6) {
    // ------------------------------------------------------------ P^T, dS^T
    const int rq = warp & 3;
    const int grp = (warp - 6) >> 2;     // queries [16 grp, 16 grp + 16) of each block
    const int row = rq * 32 + lane;      // key within the block (= TMEM lane)
    const int key = kv0 + row;
    const uint32_t lane_addr = static_cast<uint32_t>(rq * 32) << 16;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int b = it & 1;
      const float* lse_h = p.lse + head_row(it) * p.stride + row_base;
      const float* d_h = p.dsum + head_row(it) * p.stride + row_base;
      const bool got =
          mbar_wait(bar(AB_SDP + b), (it >> 1) & 1, abort_flag) &&
          (!p.ld_bulk || mbar_wait(bar(AB_LDFULL + b), (it >> 1) & 1, abort_flag)) &&
          // dS^T buffer b is free once dK and dQ^T of block it - 2 are done
          (it < 2 || mbar_wait(bar(AB_DQFULL + b), ((it - 2) >> 1) & 1, abort_flag));
      // the warp leaves together (the TMEM accesses below are warp-collective)
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int i = step_block(it);
      const int q0 = i * AB_BQ;
      const bool need_mask =
          (p.causal && q0 < kv0 + AB_BK) || q0 + AB_BQ > p.seq || kv0 + AB_BK > p.seq;
      const uint32_t tS = tmem + lane_addr + 128u * b, tP = tS + 64u;
      const uint32_t s_lse = s0 + AOFF_LD + b * (2 * AB_BQ * 4), s_d = s_lse + AB_BQ * 4;
      const uint32_t ds_row = s0 + AOFF_DS + b * AB_DSTILE + static_cast<uint32_t>(row) * 128u;
      {
        // this thread's 16 queries [16 grp, 16 grp + 16): one TMEM round trip
        const int c0 = grp * 16;
        uint32_t sv[16], dv[16];
        tmem_ld_32x32b_x16(tS + c0, sv);
        tmem_ld_32x32b_x16(tP + c0, dv);
        tmem_ld_wait();
        uint32_t pk[8], dk[8];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          // lse and D of these 4 queries: the same for every key thread
          float4 l4, d4;
          if (p.ld_bulk) {
            l4 = ld_shared_v4f(s_lse + (c0 + e) * 4);
            d4 = ld_shared_v4f(s_d + (c0 + e) * 4);
          } else {
            const float* lp = lse_h + q0 + c0 + e;
            const float* dp = d_h + q0 + c0 + e;
            l4 = make_float4(__ldg(lp), __ldg(lp + 1), __ldg(lp + 2), __ldg(lp + 3));
            d4 = make_float4(__ldg(dp), __ldg(dp + 1), __ldg(dp + 2), __ldg(dp + 3));
          }
          const float lq[4] = {l4.x, l4.y, l4.z, l4.w};
          const float dq[4] = {d4.x, d4.y, d4.z, d4.w};
          float pp[4], ds[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float pv = ex2_approx(fmaf(__uint_as_float(sv[e + u]), sl2, -lq[u]));
            const float dsv = pv * (__uint_as_float(dv[e + u]) - dq[u]);
            if (need_mask) {
              const int q = q0 + c0 + e + u;
              const bool valid = key < p.seq && q < p.seq && (!p.causal || q >= key);
              pp[u] = valid ? pv : 0.f;
              ds[u] = valid ? dsv : 0.f;
            } else {
              pp[u] = pv;
              ds[u] = dsv;
            }
          }
          pk[e >> 1] = pack_bf16x2(pp[0], pp[1]);
          pk[(e >> 1) + 1] = pack_bf16x2(pp[2], pp[3]);
          dk[e >> 1] = pack_bf16x2(ds[0], ds[1]);
          dk[(e >> 1) + 1] = pack_bf16x2(ds[2], ds[3]);
        }
        // P^T of the 16 queries into the first 8 of the 16 S^T columns this
        // thread has read
        tmem_st_32x32b_x8(tS + c0, pk);
        // dS^T row `row`, queries [16 grp, 16 grp + 16): two 16-byte chunks
        // of the 128-byte swizzled row
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const uint32_t chunk = static_cast<uint32_t>(grp * 2 + u);
          st_shared_v4(ds_row + ((chunk ^ (static_cast<uint32_t>(row) & 7u)) << 4), dk[4 * u],
                       dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
        }
      }
      tmem_st_wait();
      fence_proxy_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(AB_DS + b));
        if (p.ld_bulk) mbar_arrive(bar(AB_LDEMPTY + b));
      }
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, ERR_WAIT_ATTN);
      *abort_flag = 1;
    } else if (__all_sync(0xffffffffu, mbar_wait(bar(AB_DONE), 0, abort_flag))) {
      tc_fence_after();
      // tcgen05.ld is warp-collective: every lane loads. The warp's 32 keys x
      // 32 columns of dK (scaled) and of dV go to its two 2 KB tiles in the Q
      // ring (idle once every MMA is done), 64-byte rows, and leave with two
      // TMA stores when all 32 keys are inside the sequence; otherwise the
      // keys inside it are stored directly.
      const uint32_t tile = s0 + AOFF_Q + static_cast<uint32_t>(grp * 4 + rq) * 4096u;
      const uint32_t trow = tile + static_cast<uint32_t>(lane) * 64u;
      const bool box_inside = kv0 + rq * 32 + 32 <= p.seq;
      uint16_t* base = p.dqkv + (static_cast<int64_t>(g) * p.M + row_base + key) * p.ld +
                       p.q_w + kvh * AB_D + grp * 32;  // dK here, dV kvl x 128 columns further
      uint32_t v[2][32];  // dK, dV: both loads in flight before the wait
      tmem_ld_32x32b_x32(tmem + lane_addr + 384u + grp * 32, v[0]);
      tmem_ld_32x32b_x32(tmem + lane_addr + 256u + grp * 32, v[1]);
      tmem_ld_wait();
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {  // dK, then dV
        const float sc = kv == 0 ? p.scale : 1.f;
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(v[kv][2 * e]) * sc,
                             __uint_as_float(v[kv][2 * e + 1]) * sc);
        if (box_inside) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            st_shared_v4(trow + kv * 2048u + (static_cast<uint32_t>(u) << 4), w[4 * u],
                         w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        } else if (key < p.seq) {
          uint4* dst = reinterpret_cast<uint4*>(base + kv * p.kvl * AB_D);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            dst[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      }
      if (box_inside) {
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
          const int col = p.q_w + kvh * AB_D + grp * 32;
          const int trow0 = row_base + kv0 + rq * 32;
          tma_store_3d(&tm_st, tile, col, trow0, g);
          tma_store_3d(&tm_st, tile + 2048u, col + p.kvl * AB_D, trow0, g);
          bulk_commit();
          bulk_wait_read<0>();  // the tiles are read before the CTA's shared memory goes away
        }
        __syncwarp();
      }
    } else {
      if (lane == 0) atomicOr(p.err, ERR_WAIT_ATTN);
      *abort_flag = 1;
    }
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------ dQ^T
    const int rq = warp & 3;
    const int dcol = rq * 32 + lane;  // head-dimension column (= TMEM lane)
    const uint32_t lane_addr = static_cast<uint32_t>(rq * 32) << 16;
    // accumulator rows [stride][128]: a warp's 32 lanes cover 128 contiguous bytes
    bool ok = true;
    for (int it = 0; ok && it < n_it; ++it) {
      const int b = it & 1;
      // the warp leaves together (the TMEM loads are warp-collective)
      if (!__all_sync(0xffffffffu, mbar_wait(bar(AB_DQFULL + b), (it >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[AB_BQ];
      const uint32_t tP = tmem + lane_addr + 128u * b + 64u;
      tmem_ld_32x32b_x32(tP, &v[0]);
      tmem_ld_32x32b_x32(tP + 32, &v[32]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(bar(AB_DQEMPTY + b));  // the columns may be overwritten now
      const int q0 = step_block(it) * AB_BQ;
      const int nq_valid = min(AB_BQ, p.seq - q0);
      float* a = p.dq_acc + (head_row(it) * p.stride + row_base + q0) * AB_D + dcol;
#pragma unroll
      for (int q = 0; q < AB_BQ; ++q)
        if (q < nq_valid) red_add_f32(a + static_cast<int64_t>(q) * AB_D, v[q]);
    }
    if (!ok) {
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

// Before the main kernel: D[(shard, head)][token] = sum_d dO * O over the
// head's 128 columns (fp32), and the token's row of the dQ accumulator
// zeroed. 16 threads per (shard, token, head), 8 columns each.
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(
    const uint16_t* __restrict__ O, const uint16_t* __restrict__ dO, float* __restrict__ dsum,
    float* __restrict__ dq_acc, int64_t n_units, int hps, int64_t M, int64_t stride) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t u = i >> 4;
  const int c8 = static_cast<int>(i & 15);
  float s = 0.f;
  int64_t hb = 0, tok = 0;
  if (u < n_units) {
    const int head = static_cast<int>(u % hps);
    const int64_t gr = u / hps;  // shard * M + token
    const int64_t g = gr / M;
    tok = gr % M;
    hb = g * hps + head;
    const int64_t off = gr * (static_cast<int64_t>(hps) * AB_D) + head * AB_D + c8 * 8;
    const uint4 o = __ldg(reinterpret_cast<const uint4*>(O + off));
    const uint4 d = __ldg(reinterpret_cast<const uint4*>(dO + off));
    s = bf16_lo(o.x) * bf16_lo(d.x);
    s = fmaf(bf16_hi(o.x), bf16_hi(d.x), s);
    s = fmaf(bf16_lo(o.y), bf16_lo(d.y), s);
    s = fmaf(bf16_hi(o.y), bf16_hi(d.y), s);
    s = fmaf(bf16_lo(o.z), bf16_lo(d.z), s);
    s = fmaf(bf16_hi(o.z), bf16_hi(d.z), s);
    s = fmaf(bf16_lo(o.w), bf16_lo(d.w), s);
    s = fmaf(bf16_hi(o.w), bf16_hi(d.w), s);
    float4* acc = reinterpret_cast<float4*>(dq_acc + (hb * stride + tok) * AB_D + c8 * 8);
    acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // the 16 threads of a unit are 16 consecutive lanes of one warp
#pragma unroll
  for (int k = 8; k >= 1; k >>= 1) s += __shfl_xor_sync(0xffffffffu, s, k);
  if (u < n_units && c8 == 0) dsum[hb * stride + tok] = s;
}

// dQ (bf16, scaled) into the Q columns of dQKV from the [stride][128]
// accumulator; thread = ((shard, head), token, 8 columns), columns fastest.
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const float* __restrict__ acc,
                                                          uint16_t* __restrict__ dqkv, int64_t n,
                                                          int64_t M, int64_t stride, int hps,
                                                          int ld, float scale) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const int c8 = static_cast<int>(i % (AB_D / 8));
  const int64_t r = i / (AB_D / 8);
  const int64_t tok = r % M;
  const int64_t hb = r / M;
  const int head = static_cast<int>(hb % hps);
  const int64_t g = hb / hps;
  const float* a = acc + (hb * stride + tok) * AB_D + c8 * 8;
  const float4 x = *reinterpret_cast<const float4*>(a);
  const float4 y = *reinterpret_cast<const float4*>(a + 4);
  uint4 w;
  w.x = pack_bf16x2(x.x * scale, x.y * scale);
  w.y = pack_bf16x2(x.z * scale, x.w * scale);
  w.z = pack_bf16x2(y.x * scale, y.y * scale);
  w.w = pack_bf16x2(y.z * scale, y.w * scale);
  *reinterpret_cast<uint4*>(dqkv + (g * M + tok) * static_cast<int64_t>(ld) + head * AB_D +
                            c8 * 8) = w;
}

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 bwd_map_encoder() {
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

static bool encode_rows(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, const void* base,
                        int64_t cols, int64_t rows, int shards, uint32_t box_rows,
                        uint32_t box_cols = 64, bool swizzle = true) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(shards)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols * 2),
                           static_cast<cuuint64_t>(rows * cols * 2)};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int launch_attention_bwd(const void* QKV, const void* O, const void* dO, const float* lse,
                         int64_t batch, int64_t seq, int64_t n_q, int64_t kv_local, int n_shards,
                         int causal, void* dQKV, float* dsum, float* dq_acc, cudaStream_t s,
                         unsigned* err, int num_sms) {
  const int hps = static_cast<int>(n_q / n_shards);
  const int kvl = static_cast<int>(kv_local);
  const int64_t q_w = static_cast<int64_t>(hps) * AB_D;
  const int64_t ld = q_w + 2LL * kvl * AB_D;  // QKV row width per shard
  const int64_t M = batch * seq;
  const int64_t stride = M + 128;
  auto enc = bwd_map_encoder();
  if (enc == nullptr) return 1;
  CUtensorMap tm_kv, tm_q, tm_do, tm_st;
  if (!encode_rows(enc, &tm_kv, QKV, ld, M, n_shards, AB_BK)) return 1;
  if (!encode_rows(enc, &tm_q, QKV, ld, M, n_shards, AB_BQ)) return 1;
  if (!encode_rows(enc, &tm_do, dO, q_w, M, n_shards, AB_BQ)) return 1;
  // dK / dV stores: 32 keys x 32 columns, dense 64-byte rows
  if (!encode_rows(enc, &tm_st, dQKV, ld, M, n_shards, 32, 32, false)) return 1;

  const int64_t heads_total = static_cast<int64_t>(n_shards) * hps;
  const int nq = static_cast<int>((seq + AB_BQ - 1) / AB_BQ);
  // D = rowsum(dO * O) and the dQ accumulator's token rows zeroed
  const int64_t n_units = heads_total * M;
  attn_bwd_prep_kernel<<<static_cast<unsigned>((n_units * 16 + 255) / 256), 256, 0, s>>>(
      static_cast<const uint16_t*>(O), static_cast<const uint16_t*>(dO), dsum, dq_acc, n_units,
      hps, M, stride);

  AttnBwdParams p;
  p.seq = static_cast<int>(seq);
  p.batch = static_cast<int>(batch);
  p.hps = hps;
  p.causal = causal;
  p.nq = nq;
  p.kvl = kvl;
  p.group = hps / kvl;
  p.q_w = static_cast<int>(q_w);
  p.ld = static_cast<int>(ld);
  p.M = M;
  p.stride = stride;
  p.scale = 1.0f / sqrtf(static_cast<float>(AB_D));
  p.scale_log2 = 1.4426950408889634f * p.scale;
  p.ld_bulk = (M % 4 == 0 && seq % 4 == 0) ? 1 : 0;  // 16-byte aligned lse / D rows
  p.lse = lse;
  p.dsum = dsum;
  p.dq_acc = dq_acc;
  p.dqkv = static_cast<uint16_t*>(dQKV);
  p.err = err;
  cudaFuncSetAttribute(attention_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       AB_SMEM);
  const dim3 grid(static_cast<unsigned>(static_cast<int64_t>(n_shards) * kvl * batch),
                  static_cast<unsigned>((seq + AB_BK - 1) / AB_BK));
  attention_bwd_tc_kernel<<<grid, AB_THREADS, AB_SMEM, s>>>(tm_kv, tm_q, tm_do, tm_st, p);

  const int64_t n = heads_total * M * (AB_D / 8);
  attn_bwd_dq_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(
      dq_acc, static_cast<uint16_t*>(dQKV), n, M, stride, hps, static_cast<int>(ld), p.scale);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
