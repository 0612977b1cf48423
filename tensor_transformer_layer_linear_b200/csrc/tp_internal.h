// Host-side interface between the C-ABI layer (tp_api.cu) and the kernel
// translation units. Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tpk {

enum KernelId {
  KID_SHARD = 0,
  KID_GEMM_COLUMN = 1,
  KID_GEMM_ROW = 2,
  KID_REDUCE = 3,
  KID_REDUCE_LN = 4,
  KID_LAYERNORM = 5,
  KID_ATTENTION = 6,
  KID_ALL_GATHER = 7,
  KID_GEMM_BACKWARD = 8,
  KID_ELEMENTWISE = 9,
  KID_COLSUM = 10,
  KID_ATTENTION_BWD = 11,
  KID_LAYERNORM_BWD = 12,
  KID_COUNT = 13
};

// One batched GEMM over G shards: D[g] (M x Nc) = A[g] (M x K) . B[g]^T with
// A [G_A][M][K] (G_A = G when a_batched, else 1: the replicated input) and
// B [G][Nc][K], both K-major bf16. D [G][M][Nc] is either bf16 with an
// optional bias [G][Nc] and activation, or fp32 (no bias, no activation).
//
// Backward variants: with a_mn (b_mn) the operand is MN-major, A [G_A][K][M]
// (B [G_B][K][Nc]); b_batched = false shares B across the batch; act 3 is the
// GeLU backward epilogue D = bf16(acc * aux), aux = GeLU'(Z) [G][M][Nc] bf16;
// act 4 is the forward recompute D = bf16(GeLU(acc + bias)) that also writes
// aux_out = bf16(GeLU'(acc + bias)) [G][M][Nc]. Products with an MN-major
// A write fp32; with only B MN-major, fp32 or bf16 (act 0, no bias).
struct GemmProblem {
  const void* A;
  const void* B;
  void* D;
  const void* bias;
  int M, Nc, K, G;
  bool a_batched;
  bool out_f32;
  int act;  // 0 none, 1 GeLU (erf form), 2 gated SiLU(gate) * up (D has Nc / 2 columns),
            // 3 times aux, 4 GeLU with GeLU' to aux_out
  bool b_batched = true;
  bool a_mn = false;
  bool b_mn = false;
  const void* aux = nullptr;
  void* aux_out = nullptr;
};

// Returns 0 on success, 1 if a tensor map could not be encoded, 2 if the
// launch failed (cudaGetLastError()).
int launch_gemm(const GemmProblem& p, cudaStream_t s, unsigned* err, int num_sms);

// Sequence-sharded layout of token rows (sp_n > 0): row b*S + s lives at
// [s / (S/N)][b][s % (S/N)] of [N][batch][S/N]; sp_n == 0 means token order.

// Y = sum_{i<N} P_i + bias + residual (bf16 out). n_elems % 8 == 0, h % 8 == 0.
// With sp_n > 0 the residual and Y use the sequence-sharded layout.
int launch_reduce(const float* P, int n_shards, int64_t rows, int64_t h, const void* bias,
                  const void* residual, void* Y, cudaStream_t s, int num_sms, int sp_n = 0,
                  int sp_batch = 0, int sp_seq = 0);

// X (token order) from X_shards (sequence-sharded layout).
int launch_all_gather_sequence(const void* Xs, int sp_n, int sp_batch, int sp_seq, int64_t h,
                               void* X, cudaStream_t s, int num_sms);

// Per row: S = bf16(sum_i P_i + bias + residual) -> Y_sum (if non-null);
// Y_ln = LN(S) with gamma, beta, eps (if non-null). n_shards may be 0
// (then S = residual, i.e. a plain LayerNorm of `residual`). h % 8 == 0,
// h <= 16384.
// With sp_n > 0 the residual and Y_sum use the sequence-sharded layout and
// Y_ln is written in token order if ln_natural, else sharded.
int launch_rows_sum_ln(const float* P, int n_shards, int64_t rows, int64_t h, const void* bias,
                       const void* residual, const void* gamma, const void* beta, float eps,
                       void* Y_sum, void* Y_ln, cudaStream_t s, int sp_n = 0, int sp_batch = 0,
                       int sp_seq = 0, int ln_natural = 1);

// Causal / full attention of every shard's heads, head_dim 128. Shard rows
// of QKV are [Q (n_q/N heads) | K (kv_local heads) | V (kv_local heads)];
// local query head k uses local kv head k / (n_q/N / kv_local). Returns 3 if
// the kernel was built with fewer launch registers than its warpgroup
// register split needs (it is then not launched). With lse != nullptr the
// base-2 log-sum-exp of every query's scaled scores is written to
// lse[(shard * (n_q/N) + k) * (M + 128) + token], M = batch * seq.
// num_sms: the current device's SM count (the persistent grid's size).
int launch_attention(const void* QKV, int64_t batch, int64_t seq, int64_t n_q, int64_t kv_local,
                     int n_shards, int causal, void* O, cudaStream_t s, unsigned* err,
                     int num_sms, float* lse = nullptr);

// Attention backward of every shard's heads (head_dim 128; n_q/N query heads
// and kv_local key/value heads per shard, laid out like the forward's QKV):
// dQKV (packed like QKV) from QKV, O, dO [N][M][n_q/N x 128] and the
// forward's lse. dsum [n_q][M + 128] fp32 and dq_acc [n_q][M + 128][128]
// fp32 are scratch.
int launch_attention_bwd(const void* QKV, const void* O, const void* dO, const float* lse,
                         int64_t batch, int64_t seq, int64_t n_q, int64_t kv_local, int n_shards,
                         int causal, void* dQKV, float* dsum, float* dq_acc, cudaStream_t s,
                         unsigned* err, int num_sms);

// out[i][c][r] = W[row(i, r)][col(i, c)] for the split kinds (kind 4: GQA
// QKV with n_q query and n_kv key/value heads of head_dim).
int launch_shard(const void* W, int64_t h_in, int64_t h_out, int n_shards, int kind,
                 int64_t head_dim, void* out, cudaStream_t s, int64_t n_q = 0, int64_t n_kv = 0);

// out[g][c] = sum_r X[g][r][c] (bf16 in, fp32 out) in two deterministic
// passes through partial[groups][slabs][cols], slabs <= max_slabs chosen to
// fill the GPU. cols % 8 == 0.
int launch_colsum(const void* X, int groups, int rows, int cols, float* partial, int max_slabs,
                  float* out, cudaStream_t s, int num_sms);

// out[c] = sum over s of partial[s][c] (fp32), in slab order.
int launch_slab_sum(const float* partial, int slabs, int cols, float* out, cudaStream_t s);

// LayerNorm backward fused with the sum of N fp32 partials (the gradient at
// the LN output) and a residual gradient: dx = residual + LN'(x)^T sum_i P_i
// (bf16), dgamma, dbeta (fp32). part holds 2 * max_ctas * h floats of
// per-CTA column sums. h % 8 == 0, h <= 16384. A wait that gives up sets a
// bit in *err. With sp_n > 0, x, residual
// and dx use the sequence-sharded layout (partials stay in token order).
int launch_rows_sum_ln_bwd(const float* P, int n_shards, int64_t rows, int64_t h, const void* x,
                           const void* gamma, const void* residual, float eps, void* dx,
                           float* dgamma, float* dbeta, float* part, int max_ctas,
                           cudaStream_t s, int num_sms, unsigned* err, int sp_n = 0,
                           int sp_batch = 0, int sp_seq = 0);

// One thread waits, for at most limit_ns, on an mbarrier nothing arrives on,
// then ORs ERR_WAIT_SELFTEST into *err (the bounded-wait failure path).
int launch_selftest_wait(unsigned* err, uint64_t limit_ns, cudaStream_t s);

}  // namespace tpk
