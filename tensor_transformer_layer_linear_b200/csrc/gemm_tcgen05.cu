// Column- and row-parallel projections on the 5th-generation tensor cores.
//
// One persistent, warp-specialized kernel computes every shard's GEMM in a
// single launch ("Tensor Parallelism in Large Language Models", sections
// "Column-Parallel Linear Layer" and "Row-Parallel Linear Layer": each of
// the N shards computes X W_i, resp. X_i W_i, with no exchange):
//
//   warp 0      TMA producer: 128-byte-swizzled A and B tiles (BK = 64) into
//               a ring of shared-memory stages, completion on mbarriers.
//   warp 1      owns TMEM (two fp32 accumulators of BN columns); one thread
//               issues tcgen05.mma per stage and releases the stage with
//               tcgen05.commit.
//   warps 2-9   epilogue: tcgen05.ld of the finished accumulator, then the
//               column-parallel bias + GeLU (bf16 out) or the row-parallel
//               fp32 partials, staged in swizzled shared memory and written
//               with TMA tensor stores, overlapping the next tile's
//               mainloop.
//
// CTAS = 1: one CTA per tile of 128 x BN (tcgen05 cta_group::1).
// CTAS = 2: a cluster of two CTAs per tile of 256 x 256 (cta_group::2). Each
// CTA loads its own 128 rows of A and its own 128 rows of B^T (half of the
// tile's columns) with plain (non-multicast) TMA; the leader CTA issues the
// M = 256 MMAs, which read both CTAs' shared memory and write each CTA's 128
// rows of D into that CTA's TMEM. Per SM this halves the B panel traffic
// from L2 and lets 6 pipeline stages fit beside the epilogue staging.
//
// Tiles are (shard g, m-block, n-block), m fastest, strided over the CTAs
// (pairs). Every barrier wait is bounded; on expiry the CTA records an error
// bit, stops all roles, waits for its own copies and MMAs in flight, frees
// TMEM and returns through the same exit path.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {

constexpr int BM = 128;            // accumulator rows per CTA (TMEM lanes)
constexpr int BK = 64;             // 64 bf16 = 128 bytes = one swizzle row
constexpr int kEpiWarps = 8;       // two per TMEM lane quarter, each half the columns
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxGemmDevices = 64;  // device ordinals with a cached residency count

template <int BN, int CTAS>
struct GemmCfg {
  static constexpr int kTileM = BM * CTAS;       // rows of a tile
  static constexpr int kBRows = BN / CTAS;       // B^T rows held per CTA
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = kBRows * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (CTAS == 2) ? 6 : ((BN == 256) ? 4 : 6);
  static constexpr int kTmemCols = 2 * BN;
  // epilogue staging: per epilogue warp, kStagingBufs buffers of 32 rows x 128 bytes
  static constexpr int kStagingBufs = 1;
  static constexpr int kStagingBytes = kEpiWarps * kStagingBufs * 4096;
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int kSmemBytes =
      1024 + kStages * kStageBytes + kStagingBytes + kNumBars * 8 + 16;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(CTAS == 1 || BN == 256, "pairs use 256 x 256 tiles");
};

struct GemmParams {
  int M, Nc, K, G;
  int num_m, num_n, num_k, num_tiles;
  int a_batched, b_batched;
  int act;
  const uint16_t* bias;
  const uint16_t* aux;  // EPI_MUL_AUX: the factor GeLU'(Z) [G][M][Nc] bf16
  uint16_t* aux_out;    // EPI_GELU_AUX: receives GeLU'(Z) [G][M][Nc] bf16
  float* out_f32;       // EPI_F32 with direct_store: D [G][M][Nc] fp32
  int direct_store;     // EPI_F32: write rows with coalesced st.global instead of TMA stores
  unsigned* err;
};

// Epilogue kinds: bf16 + bias + activation (column-parallel), fp32 partials
// (row-parallel), gated SiLU(gate) * up over interleaved 128-column blocks,
// the GeLU backward bf16(acc * GeLU'(Z)) with GeLU'(Z) read from aux, and the
// backward's recompute of the column layer: bf16 GeLU(Z) out, GeLU'(Z) to
// aux_out (Z = acc + bias).
enum { EPI_BF16 = 0, EPI_F32 = 1, EPI_SWIGLU = 2, EPI_MUL_AUX = 3, EPI_GELU_AUX = 4 };

__device__ __forceinline__ float silu(float x) { return x / (1.0f + __expf(-x)); }


// A_MN / B_MN: the operand is stored MN-major (its M, resp. N, index
// contiguous; K strided), as the backward products need; it is loaded as
// 64 x 64 boxes and described to the MMA as MN-major.
template <int BN, int EPI, int CTAS, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tcgen05_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmD,
                        const __grid_constant__ CUtensorMap tmE, const GemmParams p) {
  using C = GemmCfg<BN, CTAS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* tiles = smem_raw + pad;
  uint8_t* staging = tiles + C::kStages * C::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + C::kStagingBytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * C::kStages + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = (CTAS == 2) ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int first_tile = blockIdx.x / CTAS;
  const int tile_step = gridDim.x / CTAS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kEpiWarps * CTAS);  // one arrival per epilogue warp of the pair
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmD);
    if constexpr (EPI == EPI_GELU_AUX) tma_prefetch_desc(&tmE);
  }
  if (warp == 1) {
    if constexpr (CTAS == 2)
      tmem_alloc_pair(smem_u32(tmem_holder), C::kTmemCols);
    else
      tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (CTAS == 2) cluster_sync_all();  // peer barriers initialised before use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = first_tile; ok && tile < p.num_tiles; tile += tile_step) {
        const int mb = tile % p.num_m;
        const int rest = tile / p.num_m;
        const int nb = rest % p.num_n;
        const int g = rest / p.num_n;
        const int arow = mb * C::kTileM + static_cast<int>(rank) * BM;
        const int brow = nb * BN + static_cast<int>(rank) * C::kBRows;
        for (int kb = 0; kb < p.num_k; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(tiles + stage * C::kStageBytes);
          const int ga = p.a_batched ? g : 0, gb = p.b_batched ? g : 0;
          // both CTAs of a pair count their bytes on the leader's full barrier
          const uint32_t fb = (CTAS == 2) ? mapa_shared(full_bar(stage), 0) : full_bar(stage);
          if (leader)
            mbar_arrive_expect_tx(full_bar(stage), CTAS * C::kStageBytes);
          auto load = [&](uint32_t dst, const CUtensorMap* tm, int c0, int c1, int c2) {
            if constexpr (CTAS == 2)
              tma_load_3d_pair(dst, tm, fb, c0, c1, c2);
            else
              tma_load_3d(dst, tm, fb, c0, c1, c2);
          };
          if constexpr (A_MN) {
            for (int j = 0; j < BM / 64; ++j) load(sa + j * 8192, &tmA, arow + 64 * j, kb * BK, ga);
          } else {
            load(sa, &tmA, kb * BK, arow, ga);
          }
          if constexpr (B_MN) {
            for (int j = 0; j < C::kBRows / 64; ++j)
              load(sa + C::kABytes + j * 8192, &tmB, brow + 64 * j, kb * BK, gb);
          } else {
            load(sa + C::kABytes, &tmB, kb * BK, brow, gb);
          }
          ++issued;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        atomicOr(p.err, ERR_WAIT_PRODUCER);
        *abort_flag = 1;
      }
      // Every armed stage must have landed before the CTA may exit (for a
      // pair the leader's full barriers count both CTAs' bytes).
      if (leader) {
        for (int s = 0; s < C::kStages && s < issued; ++s) {
          const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
          int never = 0;
          if (!mbar_wait(full_bar(s), par, &never)) atomicOr(p.err, ERR_WAIT_DRAIN);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(C::kTileM, BN) | (A_MN ? (1u << 15) : 0u) |
                                 (B_MN ? (1u << 16) : 0u);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = first_tile; ok && tile < p.num_tiles; tile += tile_step) {
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < p.num_k; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(tiles + stage * C::kStageBytes);
          const uint32_t sb = sa + C::kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad =
                A_MN ? umma_desc_sw128_mn(sa + kk * 2048, 8192) : umma_desc_sw128(sa + kk * 32);
            const uint64_t bd =
                B_MN ? umma_desc_sw128_mn(sb + kk * 2048, 8192) : umma_desc_sw128(sb + kk * 32);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            if constexpr (CTAS == 2)
              umma_bf16_pair(d_tmem, ad, bd, idesc, accum);
            else
              umma_bf16(d_tmem, ad, bd, idesc, accum);
          }
          if constexpr (CTAS == 2)
            umma_commit_pair_mc(empty_bar(stage), 0x3);
          else
            umma_commit(empty_bar(stage));
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if constexpr (CTAS == 2)
          umma_commit_pair_mc(tfull_bar(acc), 0x3);
        else
          umma_commit(tfull_bar(acc));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) {
        atomicOr(p.err, ERR_WAIT_MMA);
        *abort_flag = 1;
      }
      // All MMAs issued by this thread must be complete before TMEM is freed.
      if constexpr (CTAS == 2)
        umma_commit_pair(drain_bar);
      else
        umma_commit(drain_bar);
      int never = 0;
      if (!mbar_wait(drain_bar, 0, &never)) atomicOr(p.err, ERR_WAIT_DRAIN);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp e (0..7) owns TMEM lanes [32 q, 32 q + 32) (q = warp % 4) = 32
    // output rows, and half h = e / 4 of the tile's columns. Per chunk of
    // columns (32 fp32 or 64 bf16 = 128 bytes per row) every thread writes
    // its row into the warp's 128-byte-swizzled staging buffer, then one lane
    // issues a TMA tensor store of the 32-row box (rows/columns outside the
    // output are clipped by the TMA unit). The next chunk's TMEM load is in
    // flight while the current chunk is converted and stored.
    constexpr bool OUT_F32 = EPI == EPI_F32;
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t sbase =
        smem_u32(staging) + static_cast<uint32_t>((warp - 2) * C::kStagingBufs * 4096);
    uint32_t chunk_ctr = 0;
    constexpr int CW = OUT_F32 ? 32 : 64;     // columns per chunk
    constexpr int NCH = (BN / 2) / CW;        // chunks per warp per tile
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = first_tile; tile < p.num_tiles; tile += tile_step) {
      const int mb = tile % p.num_m;
      const int rest = tile / p.num_m;
      const int nb = rest % p.num_n;
      const int g = rest / p.num_n;
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int row0 = mb * C::kTileM + static_cast<int>(rank) * BM + q * 32;
      const int colh = nb * BN + half * (BN / 2);
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN + half * (BN / 2));
      if constexpr (EPI == EPI_SWIGLU) {
        // tile columns [0, 128) are gate features, [128, 256) the same up
        // features; this warp forms output features [64 half, 64 half + 64)
        // of the tile's 128, i.e. columns (nb * 128 + 64 half) of the output.
        const int ocol0 = nb * (BN / 2) + half * 64;
        const uint32_t gbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(acc * BN + half * 64);
        uint32_t w[32];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          uint32_t gv[32], uv[32];
          tmem_ld_32x32b_x32(gbase + part * 32, gv);
          tmem_ld_32x32b_x32(gbase + BN / 2 + part * 32, uv);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float a = silu(__uint_as_float(gv[e])) * __uint_as_float(uv[e]);
            const float b = silu(__uint_as_float(gv[e + 1])) * __uint_as_float(uv[e + 1]);
            w[part * 16 + (e >> 1)] = pack_bf16x2(a, b);
          }
        }
        if (ocol0 < p.Nc / 2) {
          const uint32_t sbuf = sbase + (chunk_ctr % C::kStagingBufs) * 4096u;
          ++chunk_ctr;
          if (lane == 0) bulk_wait_read<C::kStagingBufs - 1>();
          __syncwarp();
          const uint32_t row_addr = sbuf + static_cast<uint32_t>(lane) * 128u;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(row_addr + ((static_cast<uint32_t>(j) ^ (lane & 7u)) << 4), w[4 * j],
                         w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tmD, sbuf, ocol0, row0, g);
            bulk_commit();
          }
        }
      } else {
      // fp32 partials: the whole 32 x 128 slice goes to registers at once and
      // the accumulator is handed back to the MMA before any store is issued,
      // so the next-but-one tile's MMAs overlap this tile's (long) stores.
      uint32_t r[OUT_F32 ? NCH : 2][CW];
      if constexpr (OUT_F32) {
#pragma unroll
        for (int c = 0; c < NCH; ++c) tmem_ld_32x32b_x32(tbase + c * CW, &r[c][0]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (CTAS == 2)
            mbar_arrive_cluster_relaxed(mapa_shared(tempty_bar(acc), 0));  // the leader's barrier
          else
            mbar_arrive_relaxed(tempty_bar(acc));
        }
      } else {
        tmem_ld_32x32b_x32(tbase, &r[0][0]);
        tmem_ld_32x32b_x32(tbase + 32, &r[0][32]);
      }
      const bool row_ok = row0 + lane < p.M;
      const int64_t aux_row = (static_cast<int64_t>(g) * p.M + row0 + lane) * p.Nc;
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        if constexpr (!OUT_F32) {
          tmem_ld_wait();  // chunk c has arrived
          if (c + 1 < NCH) {
            tmem_ld_32x32b_x32(tbase + (c + 1) * CW, &r[(c + 1) & 1][0]);
            tmem_ld_32x32b_x32(tbase + (c + 1) * CW + 32, &r[(c + 1) & 1][32]);
          }
        }
        const int col0 = colh + c * CW;
        if (col0 >= p.Nc) continue;  // warp-uniform: the whole chunk is past the edge
        const uint32_t* rc = r[OUT_F32 ? c : (c & 1)];
        uint32_t w[32];  // this thread's 128-byte row of the chunk
        uint32_t wg[(EPI == EPI_GELU_AUX) ? 32 : 1];  // and of GeLU'(Z)
        if constexpr (OUT_F32) {
#pragma unroll
          for (int e = 0; e < 32; ++e) w[e] = rc[e];
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(rc[8 * j + e]);
            const int col = col0 + 8 * j;
            if (p.bias != nullptr && col < p.Nc) {
              const uint4 bv = *reinterpret_cast<const uint4*>(
                  p.bias + static_cast<int64_t>(g) * p.Nc + col);
              v[0] += bf16_lo(bv.x); v[1] += bf16_hi(bv.x);
              v[2] += bf16_lo(bv.y); v[3] += bf16_hi(bv.y);
              v[4] += bf16_lo(bv.z); v[5] += bf16_hi(bv.z);
              v[6] += bf16_lo(bv.w); v[7] += bf16_hi(bv.w);
            }
            if (p.act == 1) {
#pragma unroll
              for (int e = 0; e < 8; ++e) v[e] = gelu_erf(v[e]);
            }
            if constexpr (EPI == EPI_MUL_AUX) {
              uint4 gz = make_uint4(0u, 0u, 0u, 0u);
              if (row_ok && col < p.Nc)
                gz = __ldcs(reinterpret_cast<const uint4*>(p.aux + aux_row + col));
              v[0] *= bf16_lo(gz.x); v[1] *= bf16_hi(gz.x);
              v[2] *= bf16_lo(gz.y); v[3] *= bf16_hi(gz.y);
              v[4] *= bf16_lo(gz.z); v[5] *= bf16_hi(gz.z);
              v[6] *= bf16_lo(gz.w); v[7] *= bf16_hi(gz.w);
            }
            if constexpr (EPI == EPI_GELU_AUX) {
              float gr[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) v[e] = gelu_erf_with_grad(v[e], &gr[e]);
              wg[4 * j + 0] = pack_bf16x2(gr[0], gr[1]);
              wg[4 * j + 1] = pack_bf16x2(gr[2], gr[3]);
              wg[4 * j + 2] = pack_bf16x2(gr[4], gr[5]);
              wg[4 * j + 3] = pack_bf16x2(gr[6], gr[7]);
            }
            w[4 * j + 0] = pack_bf16x2(v[0], v[1]);
            w[4 * j + 1] = pack_bf16x2(v[2], v[3]);
            w[4 * j + 2] = pack_bf16x2(v[4], v[5]);
            w[4 * j + 3] = pack_bf16x2(v[6], v[7]);
          }
        }
        const uint32_t sbuf = sbase + (chunk_ctr % C::kStagingBufs) * 4096u;
        ++chunk_ctr;
        const uint32_t row_addr = sbuf + static_cast<uint32_t>(lane) * 128u;
        if (OUT_F32 && p.direct_store) {
          // Transpose through the staging rows, then eight st.global.v4 per
          // lane, each writing four full 128-byte row segments.
          __syncwarp();  // the previous chunk's reads of sbuf are done
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(row_addr + ((static_cast<uint32_t>(j) ^ (lane & 7u)) << 4), w[4 * j],
                         w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          __syncwarp();
          const int u = lane & 7;
          const int col = col0 + 4 * u;
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int rr = it * 4 + (lane >> 3);
            const float4 v = ld_shared_v4f(sbuf + static_cast<uint32_t>(rr) * 128u +
                                           ((static_cast<uint32_t>(u) ^ (rr & 7u)) << 4));
            if (row0 + rr < p.M && col < p.Nc)
              __stcs(reinterpret_cast<float4*>(
                         p.out_f32 + (static_cast<int64_t>(g) * p.M + row0 + rr) * p.Nc + col),
                     v);
          }
        } else {
          if (lane == 0) bulk_wait_read<C::kStagingBufs - 1>();  // the store that last used sbuf read it
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(row_addr + ((static_cast<uint32_t>(j) ^ (lane & 7u)) << 4), w[4 * j],
                         w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tmD, sbuf, col0, row0, g);
            bulk_commit();
          }
        }
        if constexpr (EPI == EPI_GELU_AUX) {
          // the same staging rows, once the store above has read them
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(row_addr + ((static_cast<uint32_t>(j) ^ (lane & 7u)) << 4), wg[4 * j],
                         wg[4 * j + 1], wg[4 * j + 2], wg[4 * j + 3]);
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tmE, sbuf, col0, row0, g);
            bulk_commit();
          }
        }
      }
      }  // EPI
      if constexpr (!OUT_F32) {  // (fp32 partials released the accumulator above)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (CTAS == 2)
            mbar_arrive_cluster_relaxed(mapa_shared(tempty_bar(acc), 0));  // the leader's barrier
          else
            mbar_arrive_relaxed(tempty_bar(acc));
        }
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait<0>();  // every store of this warp has completed
    if (!ok) {
      if (lane == 0) atomicOr(p.err, ERR_WAIT_EPILOGUE);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  // A pair leaves together: the leader's MMAs read the peer's shared memory
  // and the peer's epilogue arrives on the leader's barriers.
  if constexpr (CTAS == 2) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CTAS == 2)
      tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else
      tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// [d2][d1][d0] tensor (bf16 or fp32), boxes of box0 x box1 x 1 with the
// 128-byte swizzle; loads read out-of-range elements as zero, stores skip them.
static bool encode_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                      uint32_t box0, uint32_t box1, bool f32 = false) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * es, d0 * d1 * es};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, int EPI, int CTAS, bool A_MN = false, bool B_MN = false>
static int launch_gemm_t(const GemmProblem& pr, cudaStream_t s, unsigned* err, int num_sms) {
  using C = GemmCfg<BN, CTAS>;
  constexpr bool OUT_F32 = EPI == EPI_F32;
  CUtensorMap tmA, tmB, tmD, tmE;
  const uint64_t ga = pr.a_batched ? pr.G : 1, gb = pr.b_batched ? pr.G : 1;
  // K-major: [g][rows][K] in boxes of 64 (K) x rows; MN-major: [g][K][rows] in 64 x 64 boxes
  if (A_MN ? !encode_3d(&tmA, pr.A, pr.M, pr.K, ga, 64, 64)
           : !encode_3d(&tmA, pr.A, pr.K, pr.M, ga, BK, BM))
    return 1;
  if (B_MN ? !encode_3d(&tmB, pr.B, pr.Nc, pr.K, gb, 64, 64)
           : !encode_3d(&tmB, pr.B, pr.K, pr.Nc, gb, BK, C::kBRows))
    return 1;
  const uint64_t out_cols = (EPI == EPI_SWIGLU) ? pr.Nc / 2 : pr.Nc;
  if (!encode_3d(&tmD, pr.D, out_cols, pr.M, pr.G, OUT_F32 ? 32 : 64, 32, OUT_F32)) return 1;
  tmE = tmD;  // GeLU' output (same shape as D) for EPI_GELU_AUX only
  if (EPI == EPI_GELU_AUX && !encode_3d(&tmE, pr.aux_out, out_cols, pr.M, pr.G, 64, 32, false))
    return 1;
  GemmParams p;
  p.M = pr.M;
  p.Nc = pr.Nc;
  p.K = pr.K;
  p.G = pr.G;
  p.num_m = (pr.M + C::kTileM - 1) / C::kTileM;
  p.num_n = (pr.Nc + BN - 1) / BN;
  p.num_k = (pr.K + BK - 1) / BK;
  p.num_tiles = p.num_m * p.num_n * pr.G;
  p.a_batched = pr.a_batched ? 1 : 0;
  p.b_batched = pr.b_batched ? 1 : 0;
  p.act = pr.act;
  p.bias = static_cast<const uint16_t*>(pr.bias);
  p.aux = static_cast<const uint16_t*>(pr.aux);
  p.aux_out = static_cast<uint16_t*>(pr.aux_out);
  p.out_f32 = static_cast<float*>(pr.D);
  // With K <= 256 a tile's MMAs take under half as long as its fp32 stores;
  // there the stores from registers, which wait for no staging read-back,
  // keep more bytes in flight than one TMA store per warp.
  p.direct_store = (OUT_F32 && pr.K <= 256) ? 1 : 0;
  p.err = err;
  auto kern = gemm_tcgen05_kernel<BN, EPI, CTAS, A_MN, B_MN>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CTAS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Persistent grid: as many CTAs (pairs) as can be resident at once; pairs
  // need two free SMs of one GPC, which the occupancy query accounts for.
  // The count is cached per device ordinal (atomically: concurrent first
  // calls compute the same value).
  static std::atomic<int> resident_cache[kMaxGemmDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 2;
  int resident_units = (dev >= 0 && dev < kMaxGemmDevices)
                           ? resident_cache[dev].load(std::memory_order_relaxed)
                           : 0;
  if (resident_units == 0) {
    int n = num_sms / CTAS;
    if (CTAS > 1) {
      cfg.gridDim = dim3(static_cast<unsigned>(num_sms));
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters > 0 &&
          clusters < n)
        n = clusters;
      cudaGetLastError();
    }
    resident_units = n > 0 ? n : 1;
    if (dev >= 0 && dev < kMaxGemmDevices)
      resident_cache[dev].store(resident_units, std::memory_order_relaxed);
  }
  const int units = p.num_tiles < resident_units ? p.num_tiles : resident_units;
  cfg.gridDim = dim3(static_cast<unsigned>(units * CTAS));
  if (cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmD, tmE, p) != cudaSuccess) return 2;
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

int launch_gemm(const GemmProblem& p, cudaStream_t s, unsigned* err, int num_sms) {
  const bool wide = p.Nc > 128;
  const bool pair = wide && p.M > BM;  // 256-row tiles only when there are rows to fill them
  // backward products: 256-wide tiles, pairs when M > 128
  if (p.act == 3) {  // dZ = (dY B_i^T) GeLU'(Z): A K-major, B MN-major
    return p.M > BM ? launch_gemm_t<256, EPI_MUL_AUX, 2, false, true>(p, s, err, num_sms)
                    : launch_gemm_t<256, EPI_MUL_AUX, 1, false, true>(p, s, err, num_sms);
  }
  if (p.act == 4) {  // recompute: GeLU(X A_i + b_i) and GeLU' of it
    return p.M > BM ? launch_gemm_t<256, EPI_GELU_AUX, 2>(p, s, err, num_sms)
                    : launch_gemm_t<256, EPI_GELU_AUX, 1>(p, s, err, num_sms);
  }
  if (p.a_mn && p.b_mn) {
    return p.M > BM ? launch_gemm_t<256, EPI_F32, 2, true, true>(p, s, err, num_sms)
                    : launch_gemm_t<256, EPI_F32, 1, true, true>(p, s, err, num_sms);
  }
  if (p.b_mn && !p.out_f32) {  // dO = dY W_O,i^T in bf16: A K-major, B MN-major
    return p.M > BM ? launch_gemm_t<256, EPI_BF16, 2, false, true>(p, s, err, num_sms)
                    : launch_gemm_t<256, EPI_BF16, 1, false, true>(p, s, err, num_sms);
  }
  if (p.b_mn) {
    return p.M > BM ? launch_gemm_t<256, EPI_F32, 2, false, true>(p, s, err, num_sms)
                    : launch_gemm_t<256, EPI_F32, 1, false, true>(p, s, err, num_sms);
  }
  if (p.act == 2) {  // gated: 256-wide tiles always (128 gate + 128 up columns)
    return p.M > BM ? launch_gemm_t<256, EPI_SWIGLU, 2>(p, s, err, num_sms)
                    : launch_gemm_t<256, EPI_SWIGLU, 1>(p, s, err, num_sms);
  }
  if (p.out_f32) {
    if (pair) return launch_gemm_t<256, EPI_F32, 2>(p, s, err, num_sms);
    return wide ? launch_gemm_t<256, EPI_F32, 1>(p, s, err, num_sms)
                : launch_gemm_t<128, EPI_F32, 1>(p, s, err, num_sms);
  }
  if (pair) return launch_gemm_t<256, EPI_BF16, 2>(p, s, err, num_sms);
  return wide ? launch_gemm_t<256, EPI_BF16, 1>(p, s, err, num_sms)
              : launch_gemm_t<128, EPI_BF16, 1>(p, s, err, num_sms);
}

}  // namespace tpk
