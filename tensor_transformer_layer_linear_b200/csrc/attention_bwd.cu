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
// One CTA per (shard, sequence, head, 128-key block), 12 warps:
//   warp 0     TMA: the key block's K and V once, then the 128-query blocks'
//              Q and dO into a 2-deep ring (128-byte swizzle), straight out
//              of the QKV projection's [shard][token][3h/N] output and dO,
//              and the block's lse and D into shared memory;
//   warp 1     TMEM owner and the single MMA-issuing thread;
//   warps 4-11 two threads per key (TMEM lane), each for half of the block's
//              queries: P^T = exp2(S^T scale - lse), masked, stored as bf16
//              pairs over S^T in TMEM (the A operand of dV += P^T dO), and
//              dS^T = P^T * (dP^T - D) in bf16 into a swizzled shared tile
//              that is the K-major A operand of dK += dS^T Q and, read
//              MN-major, the A operand of dQ = dS K; warps 8-11 then drain
//              the block's dQ from TMEM (one thread per query) into an fp32
//              accumulator in global memory with vector reductions (every key
//              block of the sequence contributes to it);
//   at the end warps 4-11 write dK (scaled) and dV in bf16.
// Per query block the MMAs are S^T = K Q^T, dP^T = V dO^T, then dV, dK and
// dQ; dQ lands in dP^T's TMEM columns once the previous one is drained.
// TMEM: S^T [0, 128) with P^T packed into [0, 32) and [64, 96) (each half of
// the queries inside the columns its own threads have read), dP^T / dQ
// [128, 256), dV [256, 384), dK [384, 512). Causal key blocks start at the
// diagonal query block; the heaviest (first) key blocks launch first. Every
// barrier wait is bounded; a role that gives up records an error bit and the
// CTA leaves through the common exit after waiting (bounded) for its copies
// and MMAs in flight.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

constexpr int AB_BK = 128;        // keys per CTA
constexpr int AB_BQ = 128;        // queries per step
constexpr int AB_D = 128;         // head dim
constexpr int AB_THREADS = 384;
constexpr int AB_SUB = 128 * 128;          // [128 rows][64 cols] bf16: 16 KB
constexpr int AB_TILE = 2 * AB_SUB;        // [128][128] bf16: 32 KB
constexpr int AOFF_K = 0;
constexpr int AOFF_V = AOFF_K + AB_TILE;
constexpr int AOFF_Q = AOFF_V + AB_TILE;          // 2 stages
constexpr int AOFF_DO = AOFF_Q + 2 * AB_TILE;     // 2 stages
constexpr int AOFF_DS = AOFF_DO + 2 * AB_TILE;
constexpr int AOFF_LD = AOFF_DS + AB_TILE;      // lse[128], D[128] of the query block
constexpr int AOFF_BAR = AOFF_LD + 2 * AB_BQ * 4;
constexpr int AB_NUM_BARS = 12;
constexpr int AB_SMEM = 1024 + AOFF_BAR + AB_NUM_BARS * 8 + 16;
static_assert(AB_SMEM <= 232448, "shared memory budget");

constexpr int AB_KV = 0, AB_QFULL = 1, AB_QEMPTY = 3, AB_SDP = 5, AB_DS = 6, AB_DQFULL = 7,
              AB_DQEMPTY = 8, AB_DONE = 9, AB_LDFULL = 10;
constexpr uint32_t TC_S = 0, TC_DP = 128, TC_DV = 256, TC_DK = 384;

struct AttnBwdParams {
  int seq, batch, hps, causal, nq;
  int hs;        // columns of one projection per shard (hps x 128)
  long long M;   // tokens per shard
  long long stride;  // M + 128: per-head row length of lse, D and dq_acc
  float scale_log2, scale;
  int ld_bulk;        // lse / D rows 16-byte aligned: copied by the TMA warp
  const float* lse;   // [N * hps][stride], base 2, by token
  const float* dsum;  // D, same layout
  float* dq_acc;      // [N * hps][d / 4][stride][4]
  uint16_t* dqkv;     // [N][M][3 hs]
  unsigned* err;
};

__device__ __forceinline__ void red_add_v4(float* addr, uint32_t a, uint32_t b, uint32_t c,
                                           uint32_t d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(__uint_as_float(a)),
               "f"(__uint_as_float(b)), "f"(__uint_as_float(c)), "f"(__uint_as_float(d))
               : "memory");
}

__global__ void __launch_bounds__(AB_THREADS, 1)
    attention_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                            const __grid_constant__ CUtensorMap tm_do, const AttnBwdParams p) {
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
  const int head = y % p.hps;
  const int sidx = (y / p.hps) % p.batch;
  const int g = y / (p.hps * p.batch);
  const int j = blockIdx.y;  // key block
  const int kv0 = j * AB_BK;
  const int row_base = sidx * p.seq;
  const int i_first = p.causal ? j : 0;  // query blocks that see this key block
  const int n_it = p.nq - i_first;
  const int64_t hb = static_cast<int64_t>(g) * p.hps + head;  // (shard, head)

  if (threadIdx.x == 0) {
    mbar_init(bar(AB_KV), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(AB_QFULL + b), 1);
      mbar_init(bar(AB_QEMPTY + b), 1);
    }
    mbar_init(bar(AB_SDP), 1);
    mbar_init(bar(AB_DS), 8);       // one arrival per compute warp
    mbar_init(bar(AB_LDFULL), 1);
    mbar_init(bar(AB_DQFULL), 1);
    mbar_init(bar(AB_DQEMPTY), 4);  // one arrival per dQ warp
    mbar_init(bar(AB_DONE), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_holder), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA
    bool ok = true;
    const int kcol = p.hs + head * AB_D, vcol = 2 * p.hs + head * AB_D;
    mbar_arrive_expect_tx(bar(AB_KV), 2 * AB_TILE);
    tma_load_3d(s0 + AOFF_K, &tm_qkv, bar(AB_KV), kcol, row_base + kv0, g);
    tma_load_3d(s0 + AOFF_K + AB_SUB, &tm_qkv, bar(AB_KV), kcol + 64, row_base + kv0, g);
    tma_load_3d(s0 + AOFF_V, &tm_qkv, bar(AB_KV), vcol, row_base + kv0, g);
    tma_load_3d(s0 + AOFF_V + AB_SUB, &tm_qkv, bar(AB_KV), vcol + 64, row_base + kv0, g);
    int issued = 0, ld_issued = 0;
    const float* lse_h = p.lse + hb * p.stride + row_base;
    const float* d_h = p.dsum + hb * p.stride + row_base;
    for (int it = 0; it < n_it; ++it) {
      const int st = it & 1;
      const uint32_t ph = (it >> 1) & 1;
      if (!mbar_wait(bar(AB_QEMPTY + st), ph ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      const int q0 = (i_first + it) * AB_BQ;
      const int qrow = row_base + q0;
      const uint32_t qd = s0 + AOFF_Q + st * AB_TILE, dd = s0 + AOFF_DO + st * AB_TILE;
      mbar_arrive_expect_tx(bar(AB_QFULL + st), 2 * AB_TILE);
      tma_load_3d(qd, &tm_qkv, bar(AB_QFULL + st), head * AB_D, qrow, g);
      tma_load_3d(qd + AB_SUB, &tm_qkv, bar(AB_QFULL + st), head * AB_D + 64, qrow, g);
      tma_load_3d(dd, &tm_do, bar(AB_QFULL + st), head * AB_D, qrow, g);
      tma_load_3d(dd + AB_SUB, &tm_do, bar(AB_QFULL + st), head * AB_D + 64, qrow, g);
      ++issued;
      if (p.ld_bulk) {
        // the single lse / D buffer is free once the compute warps are done
        // with the previous query block
        if (it > 0 && !mbar_wait(bar(AB_DS), (it - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(AB_LDFULL), 2 * AB_BQ * 4);
        bulk_load(s0 + AOFF_LD, lse_h + q0, AB_BQ * 4, bar(AB_LDFULL));
        bulk_load(s0 + AOFF_LD + AB_BQ * 4, d_h + q0, AB_BQ * 4, bar(AB_LDFULL));
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
    for (int ii = (issued >= 2 ? issued - 2 : 0); ii < issued; ++ii)
      if (!mbar_wait(bar(AB_QFULL + (ii & 1)), (ii >> 1) & 1, &never))
        atomicOr(p.err, ERR_WAIT_DRAIN);
    if (ld_issued > 0 && !mbar_wait(bar(AB_LDFULL), (ld_issued - 1) & 1, &never))
      atomicOr(p.err, ERR_WAIT_DRAIN);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA
    constexpr uint32_t idesc_kk = umma_idesc_bf16_f32(AB_BK, AB_BQ);        // A, B K-major
    constexpr uint32_t idesc_kmn = umma_idesc_bf16_f32_bmn(AB_BK, AB_D);    // B MN-major
    constexpr uint32_t idesc_mnmn = idesc_kmn | (1u << 15);                 // A, B MN-major
    const uint32_t sK = s0 + AOFF_K, sV = s0 + AOFF_V, sDS = s0 + AOFF_DS;
    bool ok = mbar_wait(bar(AB_KV), 0, abort_flag);
    for (int it = 0; ok && it < n_it; ++it) {
      const int st = it & 1;
      const uint32_t ph = (it >> 1) & 1;
      if (!mbar_wait(bar(AB_QFULL + st), ph, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sQ = s0 + AOFF_Q + st * AB_TILE, sdO = s0 + AOFF_DO + st * AB_TILE;
      // S^T = K Q^T: rows = keys, columns = queries, contraction over d
#pragma unroll
      for (int kk = 0; kk < AB_D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * AB_SUB + (kk & 3) * 32;
        umma_bf16(tmem + TC_S, umma_desc_sw128(sK + off), umma_desc_sw128(sQ + off), idesc_kk,
                  kk > 0 ? 1u : 0u);
      }
      // dP^T = V dO^T, into the columns the previous dQ occupied
      if (it > 0) {
        if (!mbar_wait(bar(AB_DQEMPTY), (it - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
#pragma unroll
      for (int kk = 0; kk < AB_D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * AB_SUB + (kk & 3) * 32;
        umma_bf16(tmem + TC_DP, umma_desc_sw128(sV + off), umma_desc_sw128(sdO + off), idesc_kk,
                  kk > 0 ? 1u : 0u);
      }
      umma_commit(bar(AB_SDP));
      if (!mbar_wait(bar(AB_DS), it & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // dV += P^T dO (P^T from TMEM, contraction over queries)
#pragma unroll
      for (int kk = 0; kk < AB_BQ / 16; ++kk)
        umma_bf16_tmem_a(tmem + TC_DV, tmem + TC_S + kk * 8 + (kk >= 4 ? 32 : 0),
                         umma_desc_sw128_mn(sdO + kk * 2048, AB_SUB), idesc_kmn,
                         (it > 0 || kk > 0) ? 1u : 0u);
      // dK += dS^T Q
#pragma unroll
      for (int kk = 0; kk < AB_BQ / 16; ++kk)
        umma_bf16(tmem + TC_DK, umma_desc_sw128(sDS + (kk >> 2) * AB_SUB + (kk & 3) * 32),
                  umma_desc_sw128_mn(sQ + kk * 2048, AB_SUB), idesc_kmn,
                  (it > 0 || kk > 0) ? 1u : 0u);
      // dQ = dS K (dS read MN-major from the same tile; contraction over keys)
#pragma unroll
      for (int kk = 0; kk < AB_BK / 16; ++kk)
        umma_bf16(tmem + TC_DP, umma_desc_sw128_mn(sDS + kk * 2048, AB_SUB),
                  umma_desc_sw128_mn(sK + kk * 2048, AB_SUB), idesc_mnmn, kk > 0 ? 1u : 0u);
      umma_commit(bar(AB_DQFULL));
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
  } else if (warp >= 4) {
    // ------------------------------------------------------------ P^T, dS^T, dQ
    const int rq = warp & 3;
    const int grp = (warp - 4) >> 2;  // which half of the block's queries
    const int row = rq * 32 + lane;   // key within the block (= TMEM lane)
    const int key = kv0 + row;
    const uint32_t lane_addr = static_cast<uint32_t>(rq * 32) << 16;
    const float sl2 = p.scale_log2;
    const float* lse_h = p.lse + hb * p.stride + row_base;
    const float* d_h = p.dsum + hb * p.stride + row_base;
    const float* s_lse = reinterpret_cast<const float*>(sm + AOFF_LD);
    const float* s_d = s_lse + AB_BQ;
    const uint32_t ds_row = s0 + AOFF_DS + static_cast<uint32_t>(row) * 128u;
    float* acc_h = p.dq_acc + hb * (static_cast<int64_t>(AB_D) * p.stride) + row_base * 4LL;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      if (!mbar_wait(bar(AB_SDP), it & 1, abort_flag) ||
          (p.ld_bulk && !mbar_wait(bar(AB_LDFULL), it & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int i = i_first + it;
      const int q0 = i * AB_BQ;
      const bool need_mask =
          (p.causal && i == j) || q0 + AB_BQ > p.seq || kv0 + AB_BK > p.seq;
#pragma unroll 1
      for (int c = 2 * grp; c < 2 * grp + 2; ++c) {
        uint32_t sv[32], dv[32];
        tmem_ld_32x32b_x32(tmem + lane_addr + TC_S + c * 32, sv);
        tmem_ld_32x32b_x32(tmem + lane_addr + TC_DP + c * 32, dv);
        tmem_ld_wait();
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          // lse and D of these 4 queries: the same for every key thread
          float4 l4, d4;
          if (p.ld_bulk) {
            l4 = *reinterpret_cast<const float4*>(s_lse + c * 32 + e);
            d4 = *reinterpret_cast<const float4*>(s_d + c * 32 + e);
          } else {
            const float* lp = lse_h + q0 + c * 32 + e;
            const float* dp = d_h + q0 + c * 32 + e;
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
              const int q = q0 + c * 32 + e + u;
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
        // P^T of queries [32 c, 32 c + 32) into 16 columns this thread has
        // already read: [16 c, 16 c + 16) + 32 for the second half
        tmem_st_32x32b_x16(tmem + lane_addr + TC_S + c * 16 + grp * 32, pk);
        // dS^T row `row`, queries [32 c, 32 c + 32): 128-byte swizzled rows,
        // queries 0-63 in the first 16 KB half, 64-127 in the second
        const uint32_t half = ds_row + static_cast<uint32_t>(c >> 1) * AB_SUB;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t chunk = static_cast<uint32_t>((c & 1) * 4 + u);
          st_shared_v4(half + ((chunk ^ (static_cast<uint32_t>(row) & 7u)) << 4), dk[4 * u],
                       dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
        }
      }
      tmem_st_wait();
      fence_proxy_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(AB_DS));
      if (grp == 1) {
        // drain this block's dQ (one thread per query = TMEM lane)
        if (!mbar_wait(bar(AB_DQFULL), it & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[AB_D];
#pragma unroll
        for (int c = 0; c < AB_D / 32; ++c)
          tmem_ld_32x32b_x32(tmem + lane_addr + TC_DP + c * 32, &v[c * 32]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(AB_DQEMPTY));  // the columns may be overwritten now
        const int q = q0 + row;
        if (q < p.seq) {
          // layout [d / 4][stride][4]: a warp's 32 queries are 512 contiguous bytes
          float* a = acc_h + static_cast<int64_t>(q) * 4;
#pragma unroll
          for (int u = 0; u < AB_D / 4; ++u)
            red_add_v4(a + static_cast<int64_t>(u) * p.stride * 4, v[4 * u], v[4 * u + 1],
                       v[4 * u + 2], v[4 * u + 3]);
        }
      }
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, ERR_WAIT_ATTN);
      *abort_flag = 1;
    } else if (mbar_wait(bar(AB_DONE), 0, abort_flag)) {
      tc_fence_after();
      // tcgen05.ld is warp-collective: every lane loads, only rows inside
      // the sequence are stored; each group writes half of the 128 columns
      uint16_t* base = p.dqkv + (static_cast<int64_t>(g) * p.M + row_base + key) * (3 * p.hs) +
                       head * AB_D;
#pragma unroll 1
      for (int c = 2 * grp; c < 2 * grp + 2; ++c) {
        uint32_t kv[32], vv[32];
        tmem_ld_32x32b_x32(tmem + lane_addr + TC_DK + c * 32, kv);
        tmem_ld_32x32b_x32(tmem + lane_addr + TC_DV + c * 32, vv);
        tmem_ld_wait();
        if (key < p.seq) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint4 wk, wv;
            wk.x = pack_bf16x2(__uint_as_float(kv[8 * e + 0]) * p.scale,
                               __uint_as_float(kv[8 * e + 1]) * p.scale);
            wk.y = pack_bf16x2(__uint_as_float(kv[8 * e + 2]) * p.scale,
                               __uint_as_float(kv[8 * e + 3]) * p.scale);
            wk.z = pack_bf16x2(__uint_as_float(kv[8 * e + 4]) * p.scale,
                               __uint_as_float(kv[8 * e + 5]) * p.scale);
            wk.w = pack_bf16x2(__uint_as_float(kv[8 * e + 6]) * p.scale,
                               __uint_as_float(kv[8 * e + 7]) * p.scale);
            wv.x = pack_bf16x2(__uint_as_float(vv[8 * e + 0]), __uint_as_float(vv[8 * e + 1]));
            wv.y = pack_bf16x2(__uint_as_float(vv[8 * e + 2]), __uint_as_float(vv[8 * e + 3]));
            wv.z = pack_bf16x2(__uint_as_float(vv[8 * e + 4]), __uint_as_float(vv[8 * e + 5]));
            wv.w = pack_bf16x2(__uint_as_float(vv[8 * e + 6]), __uint_as_float(vv[8 * e + 7]));
            *reinterpret_cast<uint4*>(base + p.hs + c * 32 + 8 * e) = wk;
            *reinterpret_cast<uint4*>(base + 2 * p.hs + c * 32 + 8 * e) = wv;
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

// D[(shard, head)][token] = sum_d dO * O over the head's 128 columns (fp32),
// one warp per (shard, token, head).
__global__ void __launch_bounds__(256) attn_bwd_dsum_kernel(const uint16_t* __restrict__ O,
                                                            const uint16_t* __restrict__ dO,
                                                            float* __restrict__ dsum,
                                                            int64_t n_warps, int hps, int64_t M,
                                                            int64_t stride) {
  const int64_t w = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= n_warps) return;
  const int head = static_cast<int>(w % hps);
  const int64_t gr = w / hps;  // shard * M + token
  const int64_t g = gr / M, tok = gr % M;
  const int64_t off = gr * (static_cast<int64_t>(hps) * AB_D) + head * AB_D + lane * 4;
  const uint2 o = __ldg(reinterpret_cast<const uint2*>(O + off));
  const uint2 d = __ldg(reinterpret_cast<const uint2*>(dO + off));
  float s = bf16_lo(o.x) * bf16_lo(d.x);
  s = fmaf(bf16_hi(o.x), bf16_hi(d.x), s);
  s = fmaf(bf16_lo(o.y), bf16_lo(d.y), s);
  s = fmaf(bf16_hi(o.y), bf16_hi(d.y), s);
#pragma unroll
  for (int k = 16; k >= 1; k >>= 1) s += __shfl_xor_sync(0xffffffffu, s, k);
  if (lane == 0) dsum[(g * hps + head) * stride + tok] = s;
}

__global__ void __launch_bounds__(256) zero_f32x4_kernel(float4* __restrict__ p, int64_t n4) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dQ (bf16, scaled) into the Q columns of dQKV from the [d/4][stride][4]
// accumulator; thread = ((shard, head), 8 columns, token), tokens fastest.
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const float* __restrict__ acc,
                                                          uint16_t* __restrict__ dqkv, int64_t n,
                                                          int64_t M, int64_t stride, int hps,
                                                          int hs, float scale) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const int64_t tok = i % M;
  const int64_t r = i / M;
  const int c8 = static_cast<int>(r % (AB_D / 8));
  const int64_t hb = r / (AB_D / 8);
  const int head = static_cast<int>(hb % hps);
  const int64_t g = hb / hps;
  const float* a = acc + (hb * (AB_D / 4) + 2 * c8) * stride * 4 + tok * 4;
  const float4 x = *reinterpret_cast<const float4*>(a);
  const float4 y = *reinterpret_cast<const float4*>(a + stride * 4);
  uint4 w;
  w.x = pack_bf16x2(x.x * scale, x.y * scale);
  w.y = pack_bf16x2(x.z * scale, x.w * scale);
  w.z = pack_bf16x2(y.x * scale, y.y * scale);
  w.w = pack_bf16x2(y.z * scale, y.w * scale);
  *reinterpret_cast<uint4*>(dqkv + (g * M + tok) * (3 * static_cast<int64_t>(hs)) + head * AB_D +
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
                        int64_t cols, int64_t rows, int shards) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(shards)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols * 2),
                           static_cast<cuuint64_t>(rows * cols * 2)};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int launch_attention_bwd(const void* QKV, const void* O, const void* dO, const float* lse,
                         int64_t batch, int64_t seq, int64_t n_heads, int n_shards, int causal,
                         void* dQKV, float* dsum, float* dq_acc, cudaStream_t s, unsigned* err,
                         int num_sms) {
  const int hps = static_cast<int>(n_heads / n_shards);
  const int64_t hs = static_cast<int64_t>(hps) * AB_D;
  const int64_t M = batch * seq;
  const int64_t stride = M + 128;
  auto enc = bwd_map_encoder();
  if (enc == nullptr) return 1;
  CUtensorMap tm_qkv, tm_do;
  if (!encode_rows(enc, &tm_qkv, QKV, 3 * hs, M, n_shards)) return 1;
  if (!encode_rows(enc, &tm_do, dO, hs, M, n_shards)) return 1;

  const int64_t heads_total = static_cast<int64_t>(n_shards) * hps;
  // dQ accumulator to zero, D = rowsum(dO * O)
  const int64_t n4 = heads_total * AB_D * stride / 4;
  int64_t zb = (n4 + 255) / 256;
  if (zb > 8LL * num_sms) zb = 8LL * num_sms;
  zero_f32x4_kernel<<<static_cast<unsigned>(zb), 256, 0, s>>>(reinterpret_cast<float4*>(dq_acc), n4);
  const int64_t n_warps = static_cast<int64_t>(n_shards) * M * hps;
  attn_bwd_dsum_kernel<<<static_cast<unsigned>((n_warps * 32 + 255) / 256), 256, 0, s>>>(
      static_cast<const uint16_t*>(O), static_cast<const uint16_t*>(dO), dsum, n_warps, hps, M,
      stride);

  AttnBwdParams p;
  p.seq = static_cast<int>(seq);
  p.batch = static_cast<int>(batch);
  p.hps = hps;
  p.causal = causal;
  p.nq = static_cast<int>((seq + AB_BQ - 1) / AB_BQ);
  p.hs = static_cast<int>(hs);
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
  const dim3 grid(static_cast<unsigned>(heads_total * batch),
                  static_cast<unsigned>((seq + AB_BK - 1) / AB_BK));
  attention_bwd_tc_kernel<<<grid, AB_THREADS, AB_SMEM, s>>>(tm_qkv, tm_do, p);

  const int64_t n = heads_total * (AB_D / 8) * M;
  attn_bwd_dq_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(
      dq_acc, static_cast<uint16_t*>(dQKV), n, M, stride, hps, static_cast<int>(hs), p.scale);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // namespace tpk
