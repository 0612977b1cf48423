// The C ABI of libtp.so (declared in include/tp.h): argument checks,
// workspace carving, the order of kernel launches for the MLP, attention and
// layer blocks, the per-device error word and the launch trace.
//
// Block structure ("Tensor Parallelism in Large Language Models"):
//   MLP       ColumnParallelLinear(A) + bias + GeLU  ->  RowParallelLinear(B)
//             -> one sum of the N partials (+ b2 + residual)
//   attention ColumnParallelLinear(W_QKV, whole heads) -> local attention
//             -> RowParallelLinear(W_O) -> one sum (+ b_O + residual)
//   layer     LN1 -> attention -> sum fused with the residual and LN2
//             -> MLP -> sum (+ residual)
// so every block has exactly one reduction, as the pages require.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/tp.h"
#include "tp_internal.h"

namespace {

__device__ unsigned int g_tp_error_word;

struct DevInfo {
  bool ready = false;
  tp_status status = TP_OK;
  int num_sms = 0;
  unsigned* err = nullptr;
};

constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
DevInfo g_dev[kMaxDevices];

tp_status device_info(DevInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TP_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TP_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      return TP_ERR_CUDA;
    }
    d.num_sms = sms;
    if (major != 10) {
      d.status = TP_ERR_UNSUPPORTED;  // the kernels are built for sm_100a only
    } else {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_tp_error_word) != cudaSuccess) return TP_ERR_CUDA;
      d.err = static_cast<unsigned*>(p);
      d.status = TP_OK;
    }
    d.ready = true;
  }
  *out = d;
  return d.status;
}

// ------------------------------------------------------------------ trace
struct TraceRec {
  int kid;
  cudaEvent_t a, b;
};
std::atomic<bool> g_trace_on{false};
std::mutex g_trace_mu;
std::vector<cudaEvent_t> g_ev_pool;
std::vector<TraceRec> g_trace;
std::vector<float> g_trace_ms;
int g_trace_max = 0;
int g_trace_seen = 0;

struct TraceScope {
  cudaEvent_t end = nullptr;
  cudaStream_t s;
  TraceScope(int kid, cudaStream_t st) : s(st) {
    if (!g_trace_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_trace_mu);
    const int k = g_trace_seen++;
    if (k >= g_trace_max) return;
    TraceRec r{kid, g_ev_pool[2 * k], g_ev_pool[2 * k + 1]};
    g_trace.push_back(r);
    cudaEventRecord(r.a, s);
    end = r.b;
  }
  ~TraceScope() {
    if (end != nullptr) cudaEventRecord(end, s);
  }
};

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }
inline size_t round256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }
constexpr int64_t kIntMax = 2147483647;
constexpr int kColsumSlabs = 256;  // upper bound on the column-sum slabs

tp_status gemm_status(int rc) {
  return rc == 0 ? TP_OK : TP_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* tp_status_string(int st) {
  switch (st) {
    case TP_OK: return "TP_OK";
    case TP_ERR_NULL: return "TP_ERR_NULL: a required pointer is NULL";
    case TP_ERR_SHAPE: return "TP_ERR_SHAPE: a size is invalid or not divisible by the shard count";
    case TP_ERR_ALIGN: return "TP_ERR_ALIGN: a device pointer is not 16-byte aligned";
    case TP_ERR_WORKSPACE: return "TP_ERR_WORKSPACE: workspace too small";
    case TP_ERR_UNSUPPORTED: return "TP_ERR_UNSUPPORTED: option or device not supported (needs sm_100)";
    case TP_ERR_CUDA: return "TP_ERR_CUDA: a CUDA call failed";
    case TP_ERR_TIMEOUT: return "TP_ERR_TIMEOUT: a bounded wait inside a kernel expired";
    default: return "unknown tp_status";
  }
}

const char* tp_kernel_name(int kid) {
  switch (kid) {
    case tpk::KID_SHARD: return "shard_transpose";
    case tpk::KID_GEMM_COLUMN: return "gemm_column_parallel";
    case tpk::KID_GEMM_ROW: return "gemm_row_parallel";
    case tpk::KID_REDUCE: return "reduce_partials";
    case tpk::KID_REDUCE_LN: return "reduce_partials_layernorm";
    case tpk::KID_LAYERNORM: return "layernorm";
    case tpk::KID_ATTENTION: return "attention";
    case tpk::KID_ALL_GATHER: return "all_gather_sequence";
    case tpk::KID_GEMM_BACKWARD: return "gemm_backward";
    case tpk::KID_ELEMENTWISE: return "gelu_elementwise";
    case tpk::KID_COLSUM: return "column_sum";
    case tpk::KID_ATTENTION_BWD: return "attention_backward";
    case tpk::KID_LAYERNORM_BWD: return "reduce_partials_layernorm_backward";
    default: return "unknown";
  }
}

tp_status tp_trace_begin(int max_records) {
  if (max_records < 0) return TP_ERR_SHAPE;
  std::lock_guard<std::mutex> lk(g_trace_mu);
  while (static_cast<int>(g_ev_pool.size()) < 2 * max_records) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return TP_ERR_CUDA;
    g_ev_pool.push_back(e);
  }
  g_trace.clear();
  g_trace_ms.clear();
  g_trace_max = max_records;
  g_trace_seen = 0;
  g_trace_on.store(true);
  return TP_OK;
}

int tp_trace_end(void) {
  g_trace_on.store(false);
  cudaDeviceSynchronize();
  std::lock_guard<std::mutex> lk(g_trace_mu);
  g_trace_ms.assign(g_trace.size(), -1.f);
  for (size_t k = 0; k < g_trace.size(); ++k) {
    float ms = -1.f;
    if (cudaEventElapsedTime(&ms, g_trace[k].a, g_trace[k].b) == cudaSuccess) g_trace_ms[k] = ms;
  }
  return g_trace_seen;
}

tp_status tp_trace_record(int k, int* host_kernel_id, float* host_ms) {
  std::lock_guard<std::mutex> lk(g_trace_mu);
  if (k < 0 || k >= static_cast<int>(g_trace_ms.size())) return TP_ERR_SHAPE;
  if (host_kernel_id) *host_kernel_id = g_trace[k].kid;
  if (host_ms) *host_ms = g_trace_ms[k];
  return TP_OK;
}

tp_status tp_get_last_error(void* stream) {
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return TP_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return TP_ERR_CUDA;
  unsigned w = 0;
  if (cudaMemcpyFromSymbol(&w, g_tp_error_word, sizeof(w)) != cudaSuccess) return TP_ERR_CUDA;
  if (w != 0) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_tp_error_word, &zero, sizeof(zero)) != cudaSuccess) return TP_ERR_CUDA;
    return TP_ERR_TIMEOUT;
  }
  return TP_OK;
}

tp_status tp_selftest_wait_timeout(int64_t limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return TP_ERR_SHAPE;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  return tpk::launch_selftest_wait(d.err, static_cast<uint64_t>(limit_us) * 1000ull,
                                   as_stream(stream)) == 0
             ? TP_OK
             : TP_ERR_CUDA;
}

tp_status tp_shard_index_map(int kind, int64_t h_in, int64_t h_out, int n_shards,
                             int64_t head_dim, int32_t* host_owner, int64_t* host_local) {
  if (host_owner == nullptr || host_local == nullptr) return TP_ERR_NULL;
  if (h_in <= 0 || h_out <= 0 || n_shards <= 0) return TP_ERR_SHAPE;
  if (kind == TP_SPLIT_COLUMN) {
    if (h_out % n_shards) return TP_ERR_SHAPE;
    const int64_t w = h_out / n_shards;
    for (int64_t j = 0; j < h_out; ++j) {
      host_owner[j] = static_cast<int32_t>(j / w);
      host_local[j] = j % w;
    }
    return TP_OK;
  }
  if (kind == TP_SPLIT_ROW) {
    if (h_in % n_shards) return TP_ERR_SHAPE;
    const int64_t w = h_in / n_shards;
    for (int64_t r = 0; r < h_in; ++r) {
      host_owner[r] = static_cast<int32_t>(r / w);
      host_local[r] = r % w;
    }
    return TP_OK;
  }
  if (kind == TP_SPLIT_GATE_UP) {
    if (h_out % 2) return TP_ERR_SHAPE;
    const int64_t F = h_out / 2;
    if (F % n_shards || (F / n_shards) % 128) return TP_ERR_SHAPE;
    const int64_t fs = F / n_shards;
    for (int64_t j = 0; j < h_out; ++j) {
      const int64_t part = j / F, f = j % F, within = f % fs;
      host_owner[j] = static_cast<int32_t>(f / fs);
      host_local[j] = (within / 128) * 256 + part * 128 + within % 128;
    }
    return TP_OK;
  }
  if (kind == TP_SPLIT_QKV_HEADS) {
    if (h_out % 3 || head_dim <= 0) return TP_ERR_SHAPE;
    const int64_t h = h_out / 3;
    if (h % head_dim) return TP_ERR_SHAPE;
    const int64_t heads = h / head_dim;
    if (heads % n_shards) return TP_ERR_SHAPE;
    const int64_t hps = heads / n_shards, hs = h / n_shards;
    for (int64_t j = 0; j < h_out; ++j) {
      const int64_t part = j / h, within = j % h;
      const int64_t owner = (within / head_dim) / hps;
      host_owner[j] = static_cast<int32_t>(owner);
      host_local[j] = part * hs + (within - owner * hs);
    }
    return TP_OK;
  }
  return TP_ERR_SHAPE;
}

tp_status tp_shard_weights(const uint16_t* W, int64_t h_in, int64_t h_out, int n_shards, int kind,
                           int64_t head_dim, uint16_t* W_shards, void* stream) {
  if (W == nullptr || W_shards == nullptr) return TP_ERR_NULL;
  if (h_in <= 0 || h_out <= 0 || n_shards <= 0 || n_shards > 65535) return TP_ERR_SHAPE;
  if (kind == TP_SPLIT_COLUMN) {
    if (h_out % n_shards) return TP_ERR_SHAPE;
  } else if (kind == TP_SPLIT_ROW) {
    if (h_in % n_shards) return TP_ERR_SHAPE;
  } else if (kind == TP_SPLIT_QKV_HEADS) {
    if (h_out % 3 || head_dim <= 0 || (h_out / 3) % head_dim || ((h_out / 3) / head_dim) % n_shards)
      return TP_ERR_SHAPE;
  } else if (kind == TP_SPLIT_GATE_UP) {
    if (h_out % 2 || (h_out / 2) % n_shards || ((h_out / 2) / n_shards) % 128) return TP_ERR_SHAPE;
  } else {
    return TP_ERR_SHAPE;
  }
  const int64_t cols = (kind == TP_SPLIT_ROW) ? h_out : h_out / n_shards;
  const int64_t rows = (kind == TP_SPLIT_ROW) ? h_in / n_shards : h_in;
  if ((rows + 31) / 32 > kIntMax || (cols + 31) / 32 > 65535) return TP_ERR_SHAPE;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  TraceScope ts(tpk::KID_SHARD, as_stream(stream));
  return tpk::launch_shard(W, h_in, h_out, n_shards, kind, head_dim, W_shards, as_stream(stream)) == 0
             ? TP_OK
             : TP_ERR_CUDA;
}

tp_status tp_column_linear(const uint16_t* X, int64_t B, int64_t h_in, const uint16_t* W_shards,
                           const uint16_t* bias_shards, int64_t h_out, int n_shards, int act,
                           uint16_t* Y_shards, void* stream) {
  if (X == nullptr || W_shards == nullptr || Y_shards == nullptr) return TP_ERR_NULL;
  if (B <= 0 || h_in <= 0 || h_out <= 0 || n_shards <= 0) return TP_ERR_SHAPE;
  if (h_out % n_shards) return TP_ERR_SHAPE;
  const int64_t nc = h_out / n_shards;
  if (h_in % 8 || nc % 8) return TP_ERR_SHAPE;
  if (B > kIntMax || h_in > kIntMax || nc > kIntMax) return TP_ERR_SHAPE;
  if (act != TP_ACT_NONE && act != TP_ACT_GELU_ERF && act != TP_ACT_SWIGLU)
    return TP_ERR_UNSUPPORTED;
  if (act == TP_ACT_SWIGLU && (nc % 256 || bias_shards != nullptr)) return TP_ERR_UNSUPPORTED;
  if (!al16(X) || !al16(W_shards) || !al16(Y_shards) || (bias_shards && !al16(bias_shards)))
    return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  tpk::GemmProblem p;
  p.A = X;
  p.B = W_shards;
  p.D = Y_shards;
  p.bias = bias_shards;
  p.M = static_cast<int>(B);
  p.Nc = static_cast<int>(nc);
  p.K = static_cast<int>(h_in);
  p.G = n_shards;
  p.a_batched = false;
  p.out_f32 = false;
  p.act = act;
  TraceScope ts(tpk::KID_GEMM_COLUMN, as_stream(stream));
  return gemm_status(tpk::launch_gemm(p, as_stream(stream), d.err, d.num_sms));
}

tp_status tp_row_linear(const uint16_t* X_shards, int64_t B, int64_t h_in,
                        const uint16_t* W_shards, int64_t h_out, int n_shards, float* partials,
                        void* stream) {
  if (X_shards == nullptr || W_shards == nullptr || partials == nullptr) return TP_ERR_NULL;
  if (B <= 0 || h_in <= 0 || h_out <= 0 || n_shards <= 0) return TP_ERR_SHAPE;
  if (h_in % n_shards) return TP_ERR_SHAPE;
  const int64_t k = h_in / n_shards;
  if (k % 8 || h_out % 8) return TP_ERR_SHAPE;
  if (B > kIntMax || k > kIntMax || h_out > kIntMax) return TP_ERR_SHAPE;
  if (!al16(X_shards) || !al16(W_shards) || !al16(partials)) return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  tpk::GemmProblem p;
  p.A = X_shards;
  p.B = W_shards;
  p.D = partials;
  p.bias = nullptr;
  p.M = static_cast<int>(B);
  p.Nc = static_cast<int>(h_out);
  p.K = static_cast<int>(k);
  p.G = n_shards;
  p.a_batched = true;
  p.out_f32 = true;
  p.act = 0;
  TraceScope ts(tpk::KID_GEMM_ROW, as_stream(stream));
  return gemm_status(tpk::launch_gemm(p, as_stream(stream), d.err, d.num_sms));
}

tp_status tp_reduce_partials(const float* partials, int n_shards, int64_t B, int64_t h_out,
                             const uint16_t* bias, const uint16_t* residual, uint16_t* Y,
                             void* stream) {
  if (partials == nullptr || Y == nullptr) return TP_ERR_NULL;
  if (B <= 0 || h_out <= 0 || n_shards <= 0 || h_out % 8) return TP_ERR_SHAPE;
  if (!al16(partials) || !al16(Y) || (bias && !al16(bias)) || (residual && !al16(residual)))
    return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  TraceScope ts(tpk::KID_REDUCE, as_stream(stream));
  return tpk::launch_reduce(partials, n_shards, B, h_out, bias, residual, Y, as_stream(stream),
                            d.num_sms) == 0
             ? TP_OK
             : TP_ERR_CUDA;
}

tp_status tp_reduce_partials_layernorm(const float* partials, int n_shards, int64_t B,
                                       int64_t h_out, const uint16_t* bias,
                                       const uint16_t* residual, const uint16_t* gamma,
                                       const uint16_t* beta, float eps, uint16_t* Y_sum,
                                       uint16_t* Y_ln, void* stream) {
  if (partials == nullptr || gamma == nullptr || beta == nullptr || Y_sum == nullptr ||
      Y_ln == nullptr)
    return TP_ERR_NULL;
  if (B <= 0 || h_out <= 0 || n_shards <= 0 || h_out % 8 || h_out > 16384 || B > kIntMax)
    return TP_ERR_SHAPE;
  if (!(eps >= 0.f)) return TP_ERR_SHAPE;
  if (!al16(partials) || !al16(gamma) || !al16(beta) || !al16(Y_sum) || !al16(Y_ln) ||
      (bias && !al16(bias)) || (residual && !al16(residual)))
    return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  TraceScope ts(tpk::KID_REDUCE_LN, as_stream(stream));
  return tpk::launch_rows_sum_ln(partials, n_shards, B, h_out, bias, residual, gamma, beta, eps,
                                 Y_sum, Y_ln, as_stream(stream)) == 0
             ? TP_OK
             : TP_ERR_CUDA;
}

tp_status tp_layernorm(const uint16_t* X, int64_t B, int64_t h, const uint16_t* gamma,
                       const uint16_t* beta, float eps, uint16_t* Y, void* stream) {
  if (X == nullptr || gamma == nullptr || beta == nullptr || Y == nullptr) return TP_ERR_NULL;
  if (B <= 0 || h <= 0 || h % 8 || h > 16384 || B > kIntMax) return TP_ERR_SHAPE;
  if (!(eps >= 0.f)) return TP_ERR_SHAPE;
  if (!al16(X) || !al16(gamma) || !al16(beta) || !al16(Y)) return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  TraceScope ts(tpk::KID_LAYERNORM, as_stream(stream));
  return tpk::launch_rows_sum_ln(nullptr, 0, B, h, nullptr, X, gamma, beta, eps, nullptr, Y,
                                 as_stream(stream)) == 0
             ? TP_OK
             : TP_ERR_CUDA;
}

tp_status tp_attention(const uint16_t* QKV_shards, int64_t batch, int64_t seq, int64_t h,
                       int64_t n_heads, int causal, int n_shards, uint16_t* O_shards,
                       void* stream) {
  if (QKV_shards == nullptr || O_shards == nullptr) return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || h <= 0 || n_heads <= 0 || n_shards <= 0) return TP_ERR_SHAPE;
  if (h % n_heads || n_heads % n_shards) return TP_ERR_SHAPE;
  if (h / n_heads != 128) return TP_ERR_UNSUPPORTED;
  if (batch * seq > kIntMax || seq > kIntMax) return TP_ERR_SHAPE;
  if (static_cast<int64_t>(n_shards) * batch * (n_heads / n_shards) > 65535) return TP_ERR_SHAPE;
  if (!al16(QKV_shards) || !al16(O_shards)) return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  TraceScope ts(tpk::KID_ATTENTION, as_stream(stream));
  const int rc = tpk::launch_attention(QKV_shards, batch, seq, n_heads, n_heads / n_shards,
                                       n_shards, causal ? 1 : 0, O_shards, as_stream(stream),
                                       d.err, d.num_sms);
  return rc == 0 ? TP_OK : (rc == 3 ? TP_ERR_UNSUPPORTED : TP_ERR_CUDA);
}

// Backward-pass workspace pieces (bytes). Attention rows: per head,
// tokens + 128 (the query-block overhang), head_dim 128 (n_heads = h / 128).
static size_t mlp_bwd_bytes(size_t M, size_t H, size_t F, size_t N) {
  return 3 * round256(M * F * 2) + round256(N * M * H * 4) +
         round256(static_cast<size_t>(kColsumSlabs) * (F + H) * 4);
}
static size_t attn_core_bwd_bytes(size_t M, size_t H) {
  const size_t rows = M + 128;
  return round256(H / 128 * rows * 4) + round256(H * rows * 4);
}

// The attention backward's scratch inside a workspace of attn_core_bwd_bytes
// (n_q heads of 128 columns).
struct AttnBwdScratch {
  float* dsum;
  float* dq_acc;
};
static AttnBwdScratch attn_bwd_scratch(void* base, size_t M, size_t n_q) {
  const size_t rows = M + 128;
  uint8_t* p = static_cast<uint8_t*>(base);
  AttnBwdScratch sc;
  sc.dsum = reinterpret_cast<float*>(p);
  p += round256(n_q * rows * 4);
  sc.dq_acc = reinterpret_cast<float*>(p);
  return sc;
}
static size_t attn_bwd_bytes(size_t M, size_t H, size_t N) {
  // core + QKV, dQKV, O, dO (bf16) + lse + dX partials + column-sum slabs
  return attn_core_bwd_bytes(M, H) + 2 * round256(M * 3 * H * 2) + 2 * round256(M * H * 2) +
         round256(H / 128 * (M + 128) * 4) + round256(N * M * H * 4) +
         round256(static_cast<size_t>(kColsumSlabs) * 4 * H * 4);
}
constexpr int kLnBwdMaxCtas = 1024;  // per-CTA column sums of the LN backward
static size_t ln_bwd_bytes(size_t H) { return round256(2 * static_cast<size_t>(kLnBwdMaxCtas) * H * 4); }

size_t tp_workspace_bytes(int kind, int64_t tokens, int64_t h, int64_t ffn, int n_shards) {
  if (tokens <= 0 || h <= 0 || n_shards <= 0) return 0;
  // Every product below is at most a few terms of N*M*H*4, M*3H*2,
  // M*F*2, 256*(F+4H)*4 or (H/128)*(M+128)*4; when each factor is below
  // 2^31 and those largest products fit in 2^60 (checked here), no sum of
  // them can wrap a 64-bit size_t.
  if (tokens > kIntMax || h > kIntMax || ffn > kIntMax || ffn < 0) return 0;
  {
    const unsigned __int128 M = static_cast<uint64_t>(tokens), H = static_cast<uint64_t>(h);
    const unsigned __int128 F = static_cast<uint64_t>(ffn), N = static_cast<uint64_t>(n_shards);
    const unsigned __int128 lim = static_cast<unsigned __int128>(1) << 60;
    if (N * M * H * 4 >= lim || M * (F + 3 * H) * 2 >= lim || (M + 128) * H * 4 >= lim)
      return 0;
  }
  const size_t M = static_cast<size_t>(tokens), H = static_cast<size_t>(h);
  const size_t N = static_cast<size_t>(n_shards);
  const size_t partials = round256(N * M * H * 4);
  if (kind == TP_WS_MLP) {
    if (ffn <= 0) return 0;
    return round256(M * static_cast<size_t>(ffn) * 2) + partials;
  }
  if (kind == TP_WS_ATTN) {
    return round256(M * 3 * H * 2) + round256(M * H * 2) + partials;
  }
  if (kind == TP_WS_MLP_BWD) {
    if (ffn <= 0) return 0;
    // GeLU'(Z), H, dZ [N][M][F/N] bf16; dX partials [N][M][h] fp32; column-sum slabs
    return mlp_bwd_bytes(M, H, static_cast<size_t>(ffn), N);
  }
  if (kind == TP_WS_ATTN_CORE_BWD) return attn_core_bwd_bytes(M, H);
  if (kind == TP_WS_ATTN_BWD) return attn_bwd_bytes(M, H, N);
  if (kind == TP_WS_LN_BWD) return ln_bwd_bytes(H);
  if (kind == TP_WS_LAYER_BWD || kind == TP_WS_LAYER_BWD_SP) {
    if (ffn <= 0) return 0;
    // x1, h1, x2, dh1 + the attention part (its own partials and slabs
    // reused by the MLP) + G, H, dZ of the MLP + LN-backward column sums
    const size_t F = static_cast<size_t>(ffn);
    const size_t slabs = round256(static_cast<size_t>(kColsumSlabs) * (F + 4 * H) * 4);
    // (+ the gathered dY and dh1 under sequence parallelism)
    const size_t gathered = (kind == TP_WS_LAYER_BWD_SP) ? 2 * round256(M * H * 2) : 0;
    return 4 * round256(M * H * 2) + attn_bwd_bytes(M, H, N) + 3 * round256(M * F * 2) + slabs +
           ln_bwd_bytes(H) + gathered;
  }
  if (kind == TP_WS_LAYER || kind == TP_WS_LAYER_SP) {
    if (ffn <= 0) return 0;
    return 3 * round256(M * H * 2) + round256(M * 3 * H * 2) + round256(M * H * 2) +
           round256(M * static_cast<size_t>(ffn) * 2) + partials;
  }
  return 0;
}

// A block's output projection and its one reduction: the row-parallel GEMM
// into the N fp32 partials, then their sum with the bias and the residual.
static tp_status row_block_output(const uint16_t* X_shards, int64_t M, int64_t h_in,
                                  const uint16_t* W_shards, int64_t h_out, int n_shards,
                                  const uint16_t* bias, const uint16_t* residual, float* part,
                                  uint16_t* Y, void* stream) {
  tp_status st = tp_row_linear(X_shards, M, h_in, W_shards, h_out, n_shards, part, stream);
  if (st != TP_OK) return st;
  return tp_reduce_partials(part, n_shards, M, h_out, bias, residual, Y, stream);
}

tp_status tp_mlp_forward(const uint16_t* X, int64_t B, int64_t h, int64_t ffn, int n_shards,
                         const uint16_t* A_shards, const uint16_t* b1_shards,
                         const uint16_t* B_shards, const uint16_t* b2, const uint16_t* residual,
                         void* ws, size_t ws_bytes, uint16_t* Y, void* stream) {
  if (X == nullptr || A_shards == nullptr || B_shards == nullptr || Y == nullptr || ws == nullptr)
    return TP_ERR_NULL;
  if (B <= 0 || h <= 0 || ffn <= 0 || n_shards <= 0) return TP_ERR_SHAPE;
  if (ffn % n_shards || (ffn / n_shards) % 8 || h % 8) return TP_ERR_SHAPE;
  const size_t need = tp_workspace_bytes(TP_WS_MLP, B, h, ffn, n_shards);
  if (ws_bytes < need) return TP_ERR_WORKSPACE;
  if (!al16(ws)) return TP_ERR_ALIGN;
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* act = reinterpret_cast<uint16_t*>(w);
  float* part = reinterpret_cast<float*>(w + round256(static_cast<size_t>(B) * ffn * 2));
  tp_status st = tp_column_linear(X, B, h, A_shards, b1_shards, ffn, n_shards, TP_ACT_GELU_ERF,
                                  act, stream);
  if (st != TP_OK) return st;
  return row_block_output(act, B, ffn, B_shards, h, n_shards, b2, residual, part, Y, stream);
}

tp_status tp_mlp_forward_swiglu(const uint16_t* X, int64_t B, int64_t h, int64_t ffn,
                                int n_shards, const uint16_t* GU_shards,
                                const uint16_t* B_shards, const uint16_t* b2,
                                const uint16_t* residual, void* ws, size_t ws_bytes, uint16_t* Y,
                                void* stream) {
  if (X == nullptr || GU_shards == nullptr || B_shards == nullptr || Y == nullptr || ws == nullptr)
    return TP_ERR_NULL;
  if (B <= 0 || h <= 0 || ffn <= 0 || n_shards <= 0) return TP_ERR_SHAPE;
  if (ffn % n_shards || (ffn / n_shards) % 128 || h % 8) return TP_ERR_SHAPE;
  const size_t need = tp_workspace_bytes(TP_WS_MLP, B, h, ffn, n_shards);
  if (ws_bytes < need) return TP_ERR_WORKSPACE;
  if (!al16(ws)) return TP_ERR_ALIGN;
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* act = reinterpret_cast<uint16_t*>(w);
  float* part = reinterpret_cast<float*>(w + round256(static_cast<size_t>(B) * ffn * 2));
  tp_status st = tp_column_linear(X, B, h, GU_shards, nullptr, 2 * ffn, n_shards, TP_ACT_SWIGLU,
                                  act, stream);
  if (st != TP_OK) return st;
  return row_block_output(act, B, ffn, B_shards, h, n_shards, b2, residual, part, Y, stream);
}

tp_status tp_attn_forward(const uint16_t* X, int64_t batch, int64_t seq, int64_t h,
                          int64_t n_heads, int causal, int n_shards, const uint16_t* Wqkv_shards,
                          const uint16_t* bqkv_shards, const uint16_t* Wo_shards,
                          const uint16_t* bo, const uint16_t* residual, void* ws,
                          size_t ws_bytes, uint16_t* Y, void* stream) {
  if (X == nullptr || Wqkv_shards == nullptr || Wo_shards == nullptr || Y == nullptr ||
      ws == nullptr)
    return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || h <= 0 || n_heads <= 0 || n_shards <= 0) return TP_ERR_SHAPE;
  if (h % n_heads || n_heads % n_shards) return TP_ERR_SHAPE;
  if (h / n_heads != 128) return TP_ERR_UNSUPPORTED;
  const int64_t M = batch * seq;
  const size_t need = tp_workspace_bytes(TP_WS_ATTN, M, h, 0, n_shards);
  if (ws_bytes < need) return TP_ERR_WORKSPACE;
  if (!al16(ws)) return TP_ERR_ALIGN;
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* qkv = reinterpret_cast<uint16_t*>(w);
  w += round256(static_cast<size_t>(M) * 3 * h * 2);
  uint16_t* o = reinterpret_cast<uint16_t*>(w);
  w += round256(static_cast<size_t>(M) * h * 2);
  float* part = reinterpret_cast<float*>(w);
  tp_status st = tp_column_linear(X, M, h, Wqkv_shards, bqkv_shards, 3 * h, n_shards,
                                  TP_ACT_NONE, qkv, stream);
  if (st != TP_OK) return st;
  st = tp_attention(qkv, batch, seq, h, n_heads, causal, n_shards, o, stream);
  if (st != TP_OK) return st;
  return row_block_output(o, M, h, Wo_shards, h, n_shards, bo, residual, part, Y, stream);
}

tp_status tp_layer_forward(const uint16_t* X, int64_t batch, int64_t seq, int64_t h,
                           int64_t n_heads, int64_t ffn, int n_shards, const tp_layer_weights* w,
                           float ln_eps, void* ws, size_t ws_bytes, uint16_t* Y, void* stream) {
  if (X == nullptr || w == nullptr || Y == nullptr || ws == nullptr) return TP_ERR_NULL;
  if (w->ln1_gamma == nullptr || w->ln1_beta == nullptr || w->Wqkv_shards == nullptr ||
      w->Wo_shards == nullptr || w->ln2_gamma == nullptr || w->ln2_beta == nullptr ||
      w->A_shards == nullptr || w->B_shards == nullptr)
    return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || h <= 0 || n_heads <= 0 || ffn <= 0 || n_shards <= 0)
    return TP_ERR_SHAPE;
  if (h % n_heads || n_heads % n_shards || ffn % n_shards || (ffn / n_shards) % 8 || h % 8 ||
      h > 16384)
    return TP_ERR_SHAPE;
  if (h / n_heads != 128) return TP_ERR_UNSUPPORTED;
  const int64_t M = batch * seq;
  const size_t need = tp_workspace_bytes(TP_WS_LAYER, M, h, ffn, n_shards);
  if (ws_bytes < need) return TP_ERR_WORKSPACE;
  if (!al16(ws)) return TP_ERR_ALIGN;
  const size_t act_b = round256(static_cast<size_t>(M) * h * 2);
  uint8_t* p = static_cast<uint8_t*>(ws);
  uint16_t* x1 = reinterpret_cast<uint16_t*>(p); p += act_b;
  uint16_t* h1 = reinterpret_cast<uint16_t*>(p); p += act_b;
  uint16_t* x2 = reinterpret_cast<uint16_t*>(p); p += act_b;
  uint16_t* qkv = reinterpret_cast<uint16_t*>(p); p += round256(static_cast<size_t>(M) * 3 * h * 2);
  uint16_t* o = reinterpret_cast<uint16_t*>(p); p += act_b;
  uint16_t* a = reinterpret_cast<uint16_t*>(p); p += round256(static_cast<size_t>(M) * ffn * 2);
  float* part = reinterpret_cast<float*>(p);

  tp_status st = tp_layernorm(X, M, h, w->ln1_gamma, w->ln1_beta, ln_eps, x1, stream);
  if (st != TP_OK) return st;
  st = tp_column_linear(x1, M, h, w->Wqkv_shards, w->bqkv_shards, 3 * h, n_shards, TP_ACT_NONE,
                        qkv, stream);
  if (st != TP_OK) return st;
  st = tp_attention(qkv, batch, seq, h, n_heads, 1, n_shards, o, stream);
  if (st != TP_OK) return st;
  st = tp_row_linear(o, M, h, w->Wo_shards, h, n_shards, part, stream);
  if (st != TP_OK) return st;
  st = tp_reduce_partials_layernorm(part, n_shards, M, h, w->bo, X, w->ln2_gamma, w->ln2_beta,
                                    ln_eps, h1, x2, stream);
  if (st != TP_OK) return st;
  st = tp_column_linear(x2, M, h, w->A_shards, w->b1_shards, ffn, n_shards, TP_ACT_GELU_ERF, a,
                        stream);
  if (st != TP_OK) return st;
  return row_block_output(a, M, ffn, w->B_shards, h, n_shards, w->b2, h1, part, Y, stream);
}


tp_status tp_reduce_scatter_partials(const float* partials, int n_shards, int64_t batch,
                                     int64_t seq, int64_t h, const uint16_t* bias,
                                     const uint16_t* residual_shards, uint16_t* Y_shards,
                                     void* stream) {
  if (partials == nullptr || Y_shards == nullptr) return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || h <= 0 || n_shards <= 0 || h % 8 || seq % n_shards)
    return TP_ERR_SHAPE;
  if (batch * seq > kIntMax || seq > kIntMax) return TP_ERR_SHAPE;
  if (!al16(partials) || !al16(Y_shards) || (bias && !al16(bias)) ||
      (residual_shards && !al16(residual_shards)))
    return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  TraceScope ts(tpk::KID_REDUCE, as_stream(stream));
  return tpk::launch_reduce(partials, n_shards, batch * seq, h, bias, residual_shards, Y_shards,
                            as_stream(stream), d.num_sms, n_shards, static_cast<int>(batch),
                            static_cast<int>(seq)) == 0
             ? TP_OK
             : TP_ERR_CUDA;
}

tp_status tp_all_gather_sequence(const uint16_t* X_shards, int n_shards, int64_t batch,
                                 int64_t seq, int64_t h, uint16_t* X, void* stream) {
  if (X_shards == nullptr || X == nullptr) return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || h <= 0 || n_shards <= 0 || h % 8 || seq % n_shards)
    return TP_ERR_SHAPE;
  if (batch * seq > kIntMax || seq > kIntMax || h > kIntMax) return TP_ERR_SHAPE;
  if (!al16(X_shards) || !al16(X)) return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  TraceScope ts(tpk::KID_ALL_GATHER, as_stream(stream));
  return tpk::launch_all_gather_sequence(X_shards, n_shards, static_cast<int>(batch),
                                         static_cast<int>(seq), h, X, as_stream(stream),
                                         d.num_sms) == 0
             ? TP_OK
             : TP_ERR_CUDA;
}

tp_status tp_layer_forward_sp(const uint16_t* X_shards, int64_t batch, int64_t seq, int64_t h,
                              int64_t n_heads, int64_t ffn, int n_shards,
                              const tp_layer_weights* w, float ln_eps, void* ws, size_t ws_bytes,
                              uint16_t* Y_shards, void* stream) {
  if (X_shards == nullptr || w == nullptr || Y_shards == nullptr || ws == nullptr)
    return TP_ERR_NULL;
  if (w->ln1_gamma == nullptr || w->ln1_beta == nullptr || w->Wqkv_shards == nullptr ||
      w->Wo_shards == nullptr || w->ln2_gamma == nullptr || w->ln2_beta == nullptr ||
      w->A_shards == nullptr || w->B_shards == nullptr)
    return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || h <= 0 || n_heads <= 0 || ffn <= 0 || n_shards <= 0)
    return TP_ERR_SHAPE;
  if (h % n_heads || n_heads % n_shards || ffn % n_shards || (ffn / n_shards) % 8 || h % 8 ||
      h > 16384 || seq % n_shards)
    return TP_ERR_SHAPE;
  if (h / n_heads != 128) return TP_ERR_UNSUPPORTED;
  const int64_t M = batch * seq;
  if (M > kIntMax) return TP_ERR_SHAPE;
  const size_t need = tp_workspace_bytes(TP_WS_LAYER_SP, M, h, ffn, n_shards);
  if (ws_bytes < need) return TP_ERR_WORKSPACE;
  if (!al16(ws) || !al16(X_shards) || !al16(Y_shards)) return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  const size_t act_b = round256(static_cast<size_t>(M) * h * 2);
  uint8_t* p = static_cast<uint8_t*>(ws);
  uint16_t* x1 = reinterpret_cast<uint16_t*>(p); p += act_b;  // token order (gathered)
  uint16_t* h1 = reinterpret_cast<uint16_t*>(p); p += act_b;  // sequence-sharded
  uint16_t* x2 = reinterpret_cast<uint16_t*>(p); p += act_b;  // token order (gathered)
  uint16_t* qkv = reinterpret_cast<uint16_t*>(p); p += round256(static_cast<size_t>(M) * 3 * h * 2);
  uint16_t* o = reinterpret_cast<uint16_t*>(p); p += act_b;
  uint16_t* a = reinterpret_cast<uint16_t*>(p); p += round256(static_cast<size_t>(M) * ffn * 2);
  float* part = reinterpret_cast<float*>(p);
  cudaStream_t s = as_stream(stream);
  const int sb = static_cast<int>(batch), sq = static_cast<int>(seq);

  {  // LN1 on each shard's slice, written gathered (token order)
    TraceScope ts(tpk::KID_LAYERNORM, s);
    if (tpk::launch_rows_sum_ln(nullptr, 0, M, h, nullptr, X_shards, w->ln1_gamma, w->ln1_beta,
                                ln_eps, nullptr, x1, s, n_shards, sb, sq, 1) != 0)
      return TP_ERR_CUDA;
  }
  st = tp_column_linear(x1, M, h, w->Wqkv_shards, w->bqkv_shards, 3 * h, n_shards, TP_ACT_NONE,
                        qkv, stream);
  if (st != TP_OK) return st;
  st = tp_attention(qkv, batch, seq, h, n_heads, 1, n_shards, o, stream);
  if (st != TP_OK) return st;
  st = tp_row_linear(o, M, h, w->Wo_shards, h, n_shards, part, stream);
  if (st != TP_OK) return st;
  {  // reduce-scatter (+ b_O + sharded residual) -> h1 sharded; LN2 -> x2 gathered
    TraceScope ts(tpk::KID_REDUCE_LN, s);
    if (tpk::launch_rows_sum_ln(part, n_shards, M, h, w->bo, X_shards, w->ln2_gamma, w->ln2_beta,
                                ln_eps, h1, x2, s, n_shards, sb, sq, 1) != 0)
      return TP_ERR_CUDA;
  }
  st = tp_column_linear(x2, M, h, w->A_shards, w->b1_shards, ffn, n_shards, TP_ACT_GELU_ERF, a,
                        stream);
  if (st != TP_OK) return st;
  st = tp_row_linear(a, M, ffn, w->B_shards, h, n_shards, part, stream);
  if (st != TP_OK) return st;
  return tp_reduce_scatter_partials(part, n_shards, batch, seq, h, w->b2, h1, Y_shards, stream);
}

// ---------------------------------------------------------------- grouped-query attention
// Valid GQA sharding: n_q % N == 0, n_q % n_kv == 0, and either n_kv % N == 0
// (each shard owns n_kv/N whole groups) or N % n_kv == 0 (N > n_kv: one
// duplicated kv head per shard).
static bool gqa_ok(int64_t n_q, int64_t n_kv, int n_shards) {
  if (n_q <= 0 || n_kv <= 0 || n_shards <= 0) return false;
  if (n_q % n_shards || n_q % n_kv) return false;
  return (n_shards <= n_kv) ? (n_kv % n_shards == 0) : (n_shards % n_kv == 0);
}
static int64_t gqa_kv_local(int64_t n_kv, int n_shards) {
  return n_shards <= n_kv ? n_kv / n_shards : 1;
}

tp_status tp_shard_qkv_gqa(const uint16_t* W, int64_t h_in, int64_t n_q, int64_t n_kv,
                           int64_t head_dim, int n_shards, uint16_t* W_shards, void* stream) {
  if (W == nullptr || W_shards == nullptr) return TP_ERR_NULL;
  if (h_in <= 0 || head_dim <= 0 || n_shards > 65535 || !gqa_ok(n_q, n_kv, n_shards))
    return TP_ERR_SHAPE;
  const int64_t cols = (n_q / n_shards + 2 * gqa_kv_local(n_kv, n_shards)) * head_dim;
  if ((h_in + 31) / 32 > kIntMax || (cols + 31) / 32 > 65535) return TP_ERR_SHAPE;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  TraceScope ts(tpk::KID_SHARD, as_stream(stream));
  return tpk::launch_shard(W, h_in, (n_q + 2 * n_kv) * head_dim, n_shards, 4, head_dim, W_shards,
                           as_stream(stream), n_q, n_kv) == 0
             ? TP_OK
             : TP_ERR_CUDA;
}

tp_status tp_attention_gqa(const uint16_t* QKV_shards, int64_t batch, int64_t seq, int64_t n_q,
                           int64_t n_kv, int64_t head_dim, int causal, int n_shards,
                           uint16_t* O_shards, void* stream) {
  if (QKV_shards == nullptr || O_shards == nullptr) return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || !gqa_ok(n_q, n_kv, n_shards)) return TP_ERR_SHAPE;
  if (head_dim != 128) return TP_ERR_UNSUPPORTED;
  if (batch * seq > kIntMax || seq > kIntMax) return TP_ERR_SHAPE;
  if (static_cast<int64_t>(n_shards) * batch * (n_q / n_shards) > 65535) return TP_ERR_SHAPE;
  if (!al16(QKV_shards) || !al16(O_shards)) return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  TraceScope ts(tpk::KID_ATTENTION, as_stream(stream));
  const int rc = tpk::launch_attention(QKV_shards, batch, seq, n_q, gqa_kv_local(n_kv, n_shards),
                                       n_shards, causal ? 1 : 0, O_shards, as_stream(stream),
                                       d.err, d.num_sms);
  return rc == 0 ? TP_OK : (rc == 3 ? TP_ERR_UNSUPPORTED : TP_ERR_CUDA);
}

tp_status tp_attn_forward_gqa(const uint16_t* X, int64_t batch, int64_t seq, int64_t h,
                              int64_t n_q, int64_t n_kv, int causal, int n_shards,
                              const uint16_t* Wqkv_shards, const uint16_t* bqkv_shards,
                              const uint16_t* Wo_shards, const uint16_t* bo,
                              const uint16_t* residual, void* ws, size_t ws_bytes, uint16_t* Y,
                              void* stream) {
  if (X == nullptr || Wqkv_shards == nullptr || Wo_shards == nullptr || Y == nullptr ||
      ws == nullptr)
    return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || h <= 0 || !gqa_ok(n_q, n_kv, n_shards)) return TP_ERR_SHAPE;
  if (h % n_q || h / n_q != 128) return TP_ERR_UNSUPPORTED;
  const int64_t M = batch * seq;
  const int64_t qkv_cols = n_shards * (n_q / n_shards + 2 * gqa_kv_local(n_kv, n_shards)) * 128;
  // the attention workspace holds 3h QKV columns, which covers GQA (duplicated
  // kv heads included: N <= n_q)
  const size_t need = tp_workspace_bytes(TP_WS_ATTN, M, h, 0, n_shards);
  if (ws_bytes < need) return TP_ERR_WORKSPACE;
  if (!al16(ws)) return TP_ERR_ALIGN;
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* qkv = reinterpret_cast<uint16_t*>(w);
  w += round256(static_cast<size_t>(M) * 3 * h * 2);
  uint16_t* o = reinterpret_cast<uint16_t*>(w);
  w += round256(static_cast<size_t>(M) * h * 2);
  float* part = reinterpret_cast<float*>(w);
  tp_status st = tp_column_linear(X, M, h, Wqkv_shards, bqkv_shards, qkv_cols, n_shards,
                                  TP_ACT_NONE, qkv, stream);
  if (st != TP_OK) return st;
  st = tp_attention_gqa(qkv, batch, seq, n_q, n_kv, 128, causal, n_shards, o, stream);
  if (st != TP_OK) return st;
  return row_block_output(o, M, h, Wo_shards, h, n_shards, bo, residual, part, Y, stream);
}

// One GEMM of a backward pass over all shards (see tpk::GemmProblem).
static tp_status bwd_gemm(const DevInfo& d, cudaStream_t s, int n_shards, const void* A, bool a_b,
                          bool a_mn, const void* B, bool b_b, bool b_mn, void* D, int m, int nc,
                          int k, bool f32, int act = 0, const void* aux = nullptr,
                          const void* bias = nullptr, void* aux_out = nullptr,
                          int kid = tpk::KID_GEMM_BACKWARD) {
  tpk::GemmProblem g;
  g.A = A; g.B = B; g.D = D; g.bias = bias;
  g.M = m; g.Nc = nc; g.K = k; g.G = n_shards;
  g.a_batched = a_b; g.b_batched = b_b; g.a_mn = a_mn; g.b_mn = b_mn;
  g.out_f32 = f32; g.act = act; g.aux = aux; g.aux_out = aux_out;
  TraceScope ts(kid, s);
  return tpk::launch_gemm(g, s, d.err, d.num_sms) == 0 ? TP_OK : TP_ERR_CUDA;
}

static tp_status bwd_colsum(const DevInfo& d, cudaStream_t s, const uint16_t* X, int groups,
                            int rows, int cols, float* slabs, float* out) {
  TraceScope ts(tpk::KID_COLSUM, s);
  return tpk::launch_colsum(X, groups, rows, cols, slabs, kColsumSlabs, out, s, d.num_sms) == 0
             ? TP_OK
             : TP_ERR_CUDA;
}

struct MlpBwdBufs {
  uint16_t* G;   // GeLU'(Z) [N][M][F/N]
  uint16_t* H;   // GeLU(Z)  [N][M][F/N]
  uint16_t* dZ;  // [N][M][F/N]
  float* part;   // dX partials [N][M][h]
  float* slabs;  // column-sum scratch
};

// The MLP backward except its reduction: recompute, dZ, weight and bias
// gradients, and last the N partials dX_i = dZ_i A_i^T in b.part.
static tp_status mlp_backward_core(const DevInfo& d, cudaStream_t s, const uint16_t* X, int M,
                                   int H, int F, int n_shards, const uint16_t* A_shards,
                                   const uint16_t* b1_shards, const uint16_t* B_shards,
                                   const uint16_t* dY, const MlpBwdBufs& b, float* dA_shards,
                                   float* db1, float* dB_shards, float* db2) {
  const int fs = F / n_shards;
  // recompute the column layer: H_i = GeLU(Z_i), Z_i = X A_i + b1_i, with
  // GeLU'(Z_i) kept for the backward of the activation
  tp_status st = bwd_gemm(d, s, n_shards, X, false, false, A_shards, true, false, b.H, M, fs, H,
                          false, 4, nullptr, b1_shards, b.G, tpk::KID_GEMM_COLUMN);
  if (st != TP_OK) return st;
  // dZ_i = (dY B_i^T) * GeLU'(Z_i): dY shared; B_shards[i] = B_i^T is the MN-major operand
  st = bwd_gemm(d, s, n_shards, dY, false, false, B_shards, true, true, b.dZ, M, fs, H, false, 3,
                b.G);
  if (st != TP_OK) return st;
  // dA_i^T = dZ_i^T X (packed like A_shards), dB_i^T = dY^T H_i (packed like B_shards)
  st = bwd_gemm(d, s, n_shards, b.dZ, true, true, X, false, true, dA_shards, fs, H, M, true);
  if (st != TP_OK) return st;
  st = bwd_gemm(d, s, n_shards, dY, false, true, b.H, true, true, dB_shards, H, fs, M, true);
  if (st != TP_OK) return st;
  // bias gradients: column sums over the token rows
  st = bwd_colsum(d, s, b.dZ, n_shards, M, fs, b.slabs, db1);
  if (st != TP_OK) return st;
  st = bwd_colsum(d, s, dY, 1, M, H, b.slabs, db2);
  if (st != TP_OK) return st;
  // dX partials: dZ_i A_i^T; A_shards[i] = A_i^T is the MN-major operand
  return bwd_gemm(d, s, n_shards, b.dZ, true, false, A_shards, true, true, b.part, M, H, fs, true);
}

static MlpBwdBufs mlp_bwd_layout(void* ws, size_t M, size_t H, size_t F, size_t N) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  MlpBwdBufs b;
  const size_t act_b = round256(M * F * 2);
  b.G = reinterpret_cast<uint16_t*>(p); p += act_b;
  b.H = reinterpret_cast<uint16_t*>(p); p += act_b;
  b.dZ = reinterpret_cast<uint16_t*>(p); p += act_b;
  b.part = reinterpret_cast<float*>(p); p += round256(N * M * H * 4);
  b.slabs = reinterpret_cast<float*>(p);
  return b;
}

tp_status tp_mlp_backward(const uint16_t* X, int64_t B, int64_t h, int64_t ffn, int n_shards,
                          const uint16_t* A_shards, const uint16_t* b1_shards,
                          const uint16_t* B_shards, const uint16_t* dY, int residual, void* ws,
                          size_t ws_bytes, uint16_t* dX, float* dA_shards, float* db1,
                          float* dB_shards, float* db2, void* stream) {
  if (X == nullptr || A_shards == nullptr || B_shards == nullptr || dY == nullptr ||
      dX == nullptr || dA_shards == nullptr || db1 == nullptr || dB_shards == nullptr ||
      db2 == nullptr || ws == nullptr)
    return TP_ERR_NULL;
  if (B <= 0 || h <= 0 || ffn <= 0 || n_shards <= 0) return TP_ERR_SHAPE;
  if (ffn % n_shards || (ffn / n_shards) % 8 || h % 8) return TP_ERR_SHAPE;
  if (B > kIntMax || h > kIntMax || ffn > kIntMax) return TP_ERR_SHAPE;
  const size_t need = tp_workspace_bytes(TP_WS_MLP_BWD, B, h, ffn, n_shards);
  if (ws_bytes < need) return TP_ERR_WORKSPACE;
  if (!al16(ws) || !al16(X) || !al16(A_shards) || !al16(B_shards) || !al16(dY) || !al16(dX) ||
      !al16(dA_shards) || !al16(db1) || !al16(dB_shards) || !al16(db2) ||
      (b1_shards && !al16(b1_shards)))
    return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  const MlpBwdBufs b = mlp_bwd_layout(ws, B, h, ffn, n_shards);
  st = mlp_backward_core(d, as_stream(stream), X, static_cast<int>(B), static_cast<int>(h),
                         static_cast<int>(ffn), n_shards, A_shards, b1_shards, B_shards, dY, b,
                         dA_shards, db1, dB_shards, db2);
  if (st != TP_OK) return st;
  // the one reduction of the backward: dX = sum_i dX_i (+ dY through the residual)
  return tp_reduce_partials(b.part, n_shards, B, h, nullptr, residual ? dY : nullptr, dX, stream);
}

tp_status tp_attention_lse(const uint16_t* QKV_shards, int64_t batch, int64_t seq, int64_t h,
                           int64_t n_heads, int causal, int n_shards, uint16_t* O_shards,
                           float* lse, void* stream) {
  if (QKV_shards == nullptr || O_shards == nullptr || lse == nullptr) return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || h <= 0 || n_heads <= 0 || n_shards <= 0) return TP_ERR_SHAPE;
  if (h % n_heads || n_heads % n_shards) return TP_ERR_SHAPE;
  if (h / n_heads != 128) return TP_ERR_UNSUPPORTED;
  if (batch * seq > kIntMax || seq > kIntMax) return TP_ERR_SHAPE;
  if (static_cast<int64_t>(n_shards) * batch * (n_heads / n_shards) > 65535) return TP_ERR_SHAPE;
  if (!al16(QKV_shards) || !al16(O_shards) || !al16(lse)) return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  TraceScope ts(tpk::KID_ATTENTION, as_stream(stream));
  const int rc = tpk::launch_attention(QKV_shards, batch, seq, n_heads, n_heads / n_shards,
                                       n_shards, causal ? 1 : 0, O_shards, as_stream(stream),
                                       d.err, d.num_sms, lse);
  return rc == 0 ? TP_OK : (rc == 3 ? TP_ERR_UNSUPPORTED : TP_ERR_CUDA);
}

tp_status tp_attention_backward(const uint16_t* QKV_shards, const uint16_t* O_shards,
                                const uint16_t* dO_shards, const float* lse, int64_t batch,
                                int64_t seq, int64_t h, int64_t n_heads, int causal,
                                int n_shards, void* ws, size_t ws_bytes, uint16_t* dQKV_shards,
                                void* stream) {
  if (QKV_shards == nullptr || O_shards == nullptr || dO_shards == nullptr || lse == nullptr ||
      dQKV_shards == nullptr || ws == nullptr)
    return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || h <= 0 || n_heads <= 0 || n_shards <= 0) return TP_ERR_SHAPE;
  if (h % n_heads || n_heads % n_shards) return TP_ERR_SHAPE;
  if (h / n_heads != 128) return TP_ERR_UNSUPPORTED;
  if (batch * seq > kIntMax || seq > kIntMax) return TP_ERR_SHAPE;
  if (static_cast<int64_t>(n_shards) * batch * (n_heads / n_shards) > 0x7FFFFFFF) return TP_ERR_SHAPE;
  const int64_t M = batch * seq;
  const size_t need = tp_workspace_bytes(TP_WS_ATTN_CORE_BWD, M, h, 0, n_shards);
  if (ws_bytes < need) return TP_ERR_WORKSPACE;
  if (!al16(QKV_shards) || !al16(O_shards) || !al16(dO_shards) || !al16(lse) ||
      !al16(dQKV_shards) || !al16(ws))
    return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  const AttnBwdScratch sc = attn_bwd_scratch(ws, static_cast<size_t>(M), n_heads);
  TraceScope ts(tpk::KID_ATTENTION_BWD, as_stream(stream));
  const int rc = tpk::launch_attention_bwd(QKV_shards, O_shards, dO_shards, lse, batch, seq,
                                           n_heads, n_heads / n_shards, n_shards, causal ? 1 : 0,
                                           dQKV_shards, sc.dsum, sc.dq_acc,
                                           as_stream(stream), d.err, d.num_sms);
  return rc == 0 ? TP_OK : TP_ERR_CUDA;
}

struct AttnBwdBufs {
  void* core;      // D and the dQ accumulator
  uint16_t* qkv;   // [N][M][3h/N]: the forward's QKV
  uint16_t* dqkv;  // [N][M][3h/N]
  uint16_t* o;     // [N][M][h/N]: the forward's attention output
  uint16_t* dO;    // [N][M][h/N]
  float* lse;      // the forward's log-sum-exp
  float* part;     // dX partials [N][M][h]
  float* slabs;    // column-sum scratch
};

static AttnBwdBufs attn_bwd_layout(void* ws, size_t M, size_t H, size_t N) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  AttnBwdBufs b;
  b.core = p; p += attn_core_bwd_bytes(M, H);
  b.qkv = reinterpret_cast<uint16_t*>(p); p += round256(M * 3 * H * 2);
  b.dqkv = reinterpret_cast<uint16_t*>(p); p += round256(M * 3 * H * 2);
  b.o = reinterpret_cast<uint16_t*>(p); p += round256(M * H * 2);
  b.dO = reinterpret_cast<uint16_t*>(p); p += round256(M * H * 2);
  b.lse = reinterpret_cast<float*>(p); p += round256(H / 128 * (M + 128) * 4);
  b.part = reinterpret_cast<float*>(p); p += round256(N * M * H * 4);
  b.slabs = reinterpret_cast<float*>(p);
  return b;
}

// The attention block's backward except its reduction, with b.qkv, b.o and
// b.lse already holding the forward's values for X: dO, the head gradients,
// the weight and bias gradients, and last the N partials
// dX_i = dQKV_i W_QKV,i^T in b.part.
static tp_status attn_backward_core(const DevInfo& d, void* stream, const uint16_t* X,
                                    int64_t batch, int64_t seq, int64_t h, int64_t n_q,
                                    int64_t n_kv, int causal, int n_shards,
                                    const uint16_t* Wqkv_shards, const uint16_t* Wo_shards,
                                    const uint16_t* dY, const AttnBwdBufs& b, float* dWqkv_shards,
                                    float* dbqkv_shards, float* dWo_shards, float* dbo) {
  cudaStream_t s = as_stream(stream);
  const int M = static_cast<int>(batch * seq), H = static_cast<int>(h);
  const int hs = H / n_shards;  // query (and output) columns per shard
  const int64_t kvl = gqa_kv_local(n_kv, n_shards);
  const int qkv_w = hs + 2 * static_cast<int>(kvl) * 128;  // QKV columns per shard
  // dO_i = dY W_O,i^T; Wo_shards[i] = W_O,i^T is the MN-major operand
  tp_status st = bwd_gemm(d, s, n_shards, dY, false, false, Wo_shards, true, true, b.dO, M, hs,
                          H, false);
  if (st != TP_OK) return st;
  {
    const AttnBwdScratch sc = attn_bwd_scratch(b.core, static_cast<size_t>(M), n_q);
    TraceScope ts(tpk::KID_ATTENTION_BWD, s);
    if (tpk::launch_attention_bwd(b.qkv, b.o, b.dO, b.lse, batch, seq, n_q, kvl, n_shards,
                                  causal ? 1 : 0, b.dqkv, sc.dsum, sc.dq_acc, s, d.err,
                                  d.num_sms) != 0)
      return TP_ERR_CUDA;
  }
  // dW_QKV,i^T = dQKV_i^T X (packed like Wqkv_shards), dW_O,i^T = dY^T O_i (like Wo_shards)
  st = bwd_gemm(d, s, n_shards, b.dqkv, true, true, X, false, true, dWqkv_shards, qkv_w, H, M,
                true);
  if (st != TP_OK) return st;
  st = bwd_gemm(d, s, n_shards, dY, false, true, b.o, true, true, dWo_shards, H, hs, M, true);
  if (st != TP_OK) return st;
  st = bwd_colsum(d, s, b.dqkv, n_shards, M, qkv_w, b.slabs, dbqkv_shards);
  if (st != TP_OK) return st;
  st = bwd_colsum(d, s, dY, 1, M, H, b.slabs, dbo);
  if (st != TP_OK) return st;
  // dX partials: dQKV_i W_QKV,i^T; Wqkv_shards[i] = W_QKV,i^T is the MN-major operand
  return bwd_gemm(d, s, n_shards, b.dqkv, true, false, Wqkv_shards, true, true, b.part, M, H,
                  qkv_w, true);
}

static bool attn_bwd_shape_ok(int64_t batch, int64_t seq, int64_t h, int64_t n_heads,
                              int n_shards) {
  return batch > 0 && seq > 0 && h > 0 && n_heads > 0 && n_shards > 0 && h % n_heads == 0 &&
         n_heads % n_shards == 0 && batch * seq <= kIntMax &&
         static_cast<int64_t>(n_shards) * batch * (n_heads / n_shards) <= 65535;
}

tp_status tp_attn_backward(const uint16_t* X, int64_t batch, int64_t seq, int64_t h,
                           int64_t n_heads, int causal, int n_shards, const uint16_t* Wqkv_shards,
                           const uint16_t* bqkv_shards, const uint16_t* Wo_shards,
                           const uint16_t* dY, int residual, void* ws, size_t ws_bytes,
                           uint16_t* dX, float* dWqkv_shards, float* dbqkv_shards,
                           float* dWo_shards, float* dbo, void* stream) {
  if (X == nullptr || Wqkv_shards == nullptr || Wo_shards == nullptr || dY == nullptr ||
      dX == nullptr || dWqkv_shards == nullptr || dbqkv_shards == nullptr ||
      dWo_shards == nullptr || dbo == nullptr || ws == nullptr)
    return TP_ERR_NULL;
  if (!attn_bwd_shape_ok(batch, seq, h, n_heads, n_shards)) return TP_ERR_SHAPE;
  if (h / n_heads != 128) return TP_ERR_UNSUPPORTED;
  const int64_t M = batch * seq;
  if (ws_bytes < tp_workspace_bytes(TP_WS_ATTN_BWD, M, h, 0, n_shards)) return TP_ERR_WORKSPACE;
  if (!al16(ws) || !al16(X) || !al16(Wqkv_shards) || !al16(Wo_shards) || !al16(dY) ||
      !al16(dX) || !al16(dWqkv_shards) || !al16(dbqkv_shards) || !al16(dWo_shards) ||
      !al16(dbo) || (bqkv_shards && !al16(bqkv_shards)))
    return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  const AttnBwdBufs b = attn_bwd_layout(ws, M, h, n_shards);
  // recompute the forward: QKV_i = X W_QKV,i + b_i, O_i and the lse
  st = tp_column_linear(X, M, h, Wqkv_shards, bqkv_shards, 3 * h, n_shards, TP_ACT_NONE, b.qkv,
                        stream);
  if (st != TP_OK) return st;
  st = tp_attention_lse(b.qkv, batch, seq, h, n_heads, causal, n_shards, b.o, b.lse, stream);
  if (st != TP_OK) return st;
  st = attn_backward_core(d, stream, X, batch, seq, h, n_heads, n_heads, causal, n_shards,
                          Wqkv_shards, Wo_shards, dY, b, dWqkv_shards, dbqkv_shards, dWo_shards,
                          dbo);
  if (st != TP_OK) return st;
  // the one reduction of the block's backward: dX = sum_i dX_i (+ dY)
  return tp_reduce_partials(b.part, n_shards, M, h, nullptr, residual ? dY : nullptr, dX, stream);
}

tp_status tp_reduce_partials_layernorm_backward(const float* partials, int n_shards, int64_t B,
                                                int64_t h, const uint16_t* x,
                                                const uint16_t* gamma,
                                                const uint16_t* residual_grad, float eps,
                                                void* ws, size_t ws_bytes, uint16_t* dX,
                                                float* dgamma, float* dbeta, void* stream) {
  if (partials == nullptr || x == nullptr || gamma == nullptr || dX == nullptr ||
      dgamma == nullptr || dbeta == nullptr || ws == nullptr)
    return TP_ERR_NULL;
  if (B <= 0 || h <= 0 || n_shards <= 0 || h % 8 || h > 16384) return TP_ERR_SHAPE;
  if (ws_bytes < tp_workspace_bytes(TP_WS_LN_BWD, B, h, 0, n_shards)) return TP_ERR_WORKSPACE;
  if (!al16(partials) || !al16(x) || !al16(gamma) || !al16(dX) || !al16(dgamma) ||
      !al16(dbeta) || !al16(ws) || (residual_grad && !al16(residual_grad)))
    return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  cudaStream_t s = as_stream(stream);
  TraceScope ts(tpk::KID_LAYERNORM_BWD, s);
  return tpk::launch_rows_sum_ln_bwd(partials, n_shards, B, h, x, gamma, residual_grad, eps, dX,
                                     dgamma, dbeta, static_cast<float*>(ws), kLnBwdMaxCtas, s,
                                     d.num_sms, d.err) == 0
             ? TP_OK
             : TP_ERR_CUDA;
}

// The layer backward for token-ordered (sp == false) or sequence-sharded
// (sp == true) X, dY and dX; the GEMM and attention work always runs on
// token-ordered activations (all-gathered under sequence parallelism).
static tp_status layer_backward_impl(const uint16_t* X, int64_t batch, int64_t seq, int64_t h,
                                     int64_t n_heads, int64_t ffn, int n_shards,
                                     const tp_layer_weights* w, float ln_eps, const uint16_t* dY,
                                     void* ws, size_t ws_bytes, uint16_t* dX,
                                     const tp_layer_grads* g, void* stream, bool sp) {
  if (X == nullptr || w == nullptr || dY == nullptr || dX == nullptr || g == nullptr ||
      ws == nullptr)
    return TP_ERR_NULL;
  if (w->ln1_gamma == nullptr || w->ln1_beta == nullptr || w->Wqkv_shards == nullptr ||
      w->Wo_shards == nullptr || w->ln2_gamma == nullptr || w->ln2_beta == nullptr ||
      w->A_shards == nullptr || w->B_shards == nullptr)
    return TP_ERR_NULL;
  if (g->ln1_gamma == nullptr || g->ln1_beta == nullptr || g->Wqkv_shards == nullptr ||
      g->bqkv_shards == nullptr || g->Wo_shards == nullptr || g->bo == nullptr ||
      g->ln2_gamma == nullptr || g->ln2_beta == nullptr || g->A_shards == nullptr ||
      g->b1_shards == nullptr || g->B_shards == nullptr || g->b2 == nullptr)
    return TP_ERR_NULL;
  if (!attn_bwd_shape_ok(batch, seq, h, n_heads, n_shards) || ffn <= 0 || ffn % n_shards ||
      (ffn / n_shards) % 8 || h % 8 || h > 16384 || ffn > kIntMax || (sp && seq % n_shards))
    return TP_ERR_SHAPE;
  if (h / n_heads != 128) return TP_ERR_UNSUPPORTED;
  const int64_t M = batch * seq;
  if (ws_bytes < tp_workspace_bytes(sp ? TP_WS_LAYER_BWD_SP : TP_WS_LAYER_BWD, M, h, ffn,
                                    n_shards))
    return TP_ERR_WORKSPACE;
  if (!al16(ws) || !al16(X) || !al16(dY) || !al16(dX)) return TP_ERR_ALIGN;
  const float* grads[] = {g->ln1_gamma, g->ln1_beta, g->Wqkv_shards, g->bqkv_shards,
                          g->Wo_shards, g->bo, g->ln2_gamma, g->ln2_beta, g->A_shards,
                          g->b1_shards, g->B_shards, g->b2};
  for (const float* ptr : grads)
    if (!al16(ptr)) return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  cudaStream_t s = as_stream(stream);
  const size_t Mz = static_cast<size_t>(M), H = static_cast<size_t>(h);
  const size_t F = static_cast<size_t>(ffn);
  const size_t act_b = round256(Mz * H * 2);
  uint8_t* p = static_cast<uint8_t*>(ws);
  uint16_t* x1 = reinterpret_cast<uint16_t*>(p); p += act_b;   // token order
  uint16_t* h1 = reinterpret_cast<uint16_t*>(p); p += act_b;   // layout of X
  uint16_t* x2 = reinterpret_cast<uint16_t*>(p); p += act_b;   // token order
  uint16_t* dh1 = reinterpret_cast<uint16_t*>(p); p += act_b;  // layout of X
  AttnBwdBufs ab = attn_bwd_layout(p, Mz, H, n_shards);
  p += attn_bwd_bytes(Mz, H, n_shards);
  MlpBwdBufs mb;
  mb.G = reinterpret_cast<uint16_t*>(p); p += round256(Mz * F * 2);
  mb.H = reinterpret_cast<uint16_t*>(p); p += round256(Mz * F * 2);
  mb.dZ = reinterpret_cast<uint16_t*>(p); p += round256(Mz * F * 2);
  float* slabs = reinterpret_cast<float*>(p);
  p += round256(static_cast<size_t>(kColsumSlabs) * (F + 4 * H) * 4);
  float* lnb = reinterpret_cast<float*>(p);
  p += ln_bwd_bytes(H);
  // token-ordered dY and dh1 (all-gathered under sequence parallelism)
  const uint16_t* dYg = dY;
  const uint16_t* dh1g = dh1;
  uint16_t* gather_dY = nullptr;
  uint16_t* gather_dh1 = nullptr;
  if (sp) {
    gather_dY = reinterpret_cast<uint16_t*>(p); p += act_b;
    gather_dh1 = reinterpret_cast<uint16_t*>(p); p += act_b;
    dYg = gather_dY;
    dh1g = gather_dh1;
  }
  mb.part = ab.part;  // the two blocks' partials are used one after the other
  mb.slabs = slabs;
  ab.slabs = slabs;
  const int spn = sp ? n_shards : 0, sb = static_cast<int>(batch), sq = static_cast<int>(seq);

  // forward recompute: x1 = LN1(X), QKV, O, lse, h1 = X + Attn(x1), x2 = LN2(h1)
  {
    TraceScope ts(tpk::KID_LAYERNORM, s);
    if (tpk::launch_rows_sum_ln(nullptr, 0, M, h, nullptr, X, w->ln1_gamma, w->ln1_beta, ln_eps,
                                nullptr, x1, s, spn, sb, sq, 1) != 0)
      return TP_ERR_CUDA;
  }
  st = tp_column_linear(x1, M, h, w->Wqkv_shards, w->bqkv_shards, 3 * h, n_shards, TP_ACT_NONE,
                        ab.qkv, stream);
  if (st != TP_OK) return st;
  st = tp_attention_lse(ab.qkv, batch, seq, h, n_heads, 1, n_shards, ab.o, ab.lse, stream);
  if (st != TP_OK) return st;
  st = tp_row_linear(ab.o, M, h, w->Wo_shards, h, n_shards, ab.part, stream);
  if (st != TP_OK) return st;
  {
    TraceScope ts(tpk::KID_REDUCE_LN, s);
    if (tpk::launch_rows_sum_ln(ab.part, n_shards, M, h, w->bo, X, w->ln2_gamma, w->ln2_beta,
                                ln_eps, h1, x2, s, spn, sb, sq, 1) != 0)
      return TP_ERR_CUDA;
  }
  if (sp) {  // the backward of the forward's last reduce-scatter: gather dY
    TraceScope ts(tpk::KID_ALL_GATHER, s);
    if (tpk::launch_all_gather_sequence(dY, n_shards, sb, sq, h, gather_dY, s, d.num_sms) != 0)
      return TP_ERR_CUDA;
  }
  // MLP block: gradients and the partials of dx2; its one reduction is fused
  // with LN2's backward and the residual: dh1 = dY + LN2'(h1)^T sum_i dx2_i
  // (a reduce-scatter into the slices under sequence parallelism)
  st = mlp_backward_core(d, s, x2, static_cast<int>(M), static_cast<int>(h),
                         static_cast<int>(ffn), n_shards, w->A_shards, w->b1_shards, w->B_shards,
                         dYg, mb, g->A_shards, g->b1_shards, g->B_shards, g->b2);
  if (st != TP_OK) return st;
  {
    TraceScope ts(tpk::KID_LAYERNORM_BWD, s);
    if (tpk::launch_rows_sum_ln_bwd(mb.part, n_shards, M, h, h1, w->ln2_gamma, dY, ln_eps, dh1,
                                    g->ln2_gamma, g->ln2_beta, lnb, kLnBwdMaxCtas, s, d.num_sms,
                                    d.err, spn, sb, sq) != 0)
      return TP_ERR_CUDA;
  }
  if (sp) {  // the attention block's input gradient is needed in token order
    TraceScope ts(tpk::KID_ALL_GATHER, s);
    if (tpk::launch_all_gather_sequence(dh1, n_shards, sb, sq, h, gather_dh1, s, d.num_sms) != 0)
      return TP_ERR_CUDA;
  }
  // attention block: gradients and the partials of dx1; its one reduction is
  // fused with LN1's backward and the residual: dX = dh1 + LN1'(X)^T sum_i dx1_i
  st = attn_backward_core(d, stream, x1, batch, seq, h, n_heads, n_heads, 1, n_shards,
                          w->Wqkv_shards, w->Wo_shards, dh1g, ab, g->Wqkv_shards, g->bqkv_shards,
                          g->Wo_shards, g->bo);
  if (st != TP_OK) return st;
  TraceScope ts(tpk::KID_LAYERNORM_BWD, s);
  return tpk::launch_rows_sum_ln_bwd(ab.part, n_shards, M, h, X, w->ln1_gamma, dh1, ln_eps, dX,
                                     g->ln1_gamma, g->ln1_beta, lnb, kLnBwdMaxCtas, s, d.num_sms,
                                     d.err, spn, sb, sq) == 0
             ? TP_OK
             : TP_ERR_CUDA;
}

tp_status tp_layer_backward(const uint16_t* X, int64_t batch, int64_t seq, int64_t h,
                            int64_t n_heads, int64_t ffn, int n_shards, const tp_layer_weights* w,
                            float ln_eps, const uint16_t* dY, void* ws, size_t ws_bytes,
                            uint16_t* dX, const tp_layer_grads* g, void* stream) {
  return layer_backward_impl(X, batch, seq, h, n_heads, ffn, n_shards, w, ln_eps, dY, ws,
                             ws_bytes, dX, g, stream, false);
}

tp_status tp_layer_backward_sp(const uint16_t* X_shards, int64_t batch, int64_t seq, int64_t h,
                               int64_t n_heads, int64_t ffn, int n_shards,
                               const tp_layer_weights* w, float ln_eps, const uint16_t* dY_shards,
                               void* ws, size_t ws_bytes, uint16_t* dX_shards,
                               const tp_layer_grads* g, void* stream) {
  return layer_backward_impl(X_shards, batch, seq, h, n_heads, ffn, n_shards, w, ln_eps,
                             dY_shards, ws, ws_bytes, dX_shards, g, stream, true);
}

tp_status tp_attention_gqa_lse(const uint16_t* QKV_shards, int64_t batch, int64_t seq,
                               int64_t n_q, int64_t n_kv, int64_t head_dim, int causal,
                               int n_shards, uint16_t* O_shards, float* lse, void* stream) {
  if (QKV_shards == nullptr || O_shards == nullptr || lse == nullptr) return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || !gqa_ok(n_q, n_kv, n_shards)) return TP_ERR_SHAPE;
  if (head_dim != 128) return TP_ERR_UNSUPPORTED;
  if (batch * seq > kIntMax || seq > kIntMax) return TP_ERR_SHAPE;
  if (static_cast<int64_t>(n_shards) * batch * (n_q / n_shards) > 65535) return TP_ERR_SHAPE;
  if (!al16(QKV_shards) || !al16(O_shards) || !al16(lse)) return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  TraceScope ts(tpk::KID_ATTENTION, as_stream(stream));
  const int rc = tpk::launch_attention(QKV_shards, batch, seq, n_q, gqa_kv_local(n_kv, n_shards),
                                       n_shards, causal ? 1 : 0, O_shards, as_stream(stream),
                                       d.err, d.num_sms, lse);
  return rc == 0 ? TP_OK : (rc == 3 ? TP_ERR_UNSUPPORTED : TP_ERR_CUDA);
}

tp_status tp_attention_gqa_backward(const uint16_t* QKV_shards, const uint16_t* O_shards,
                                    const uint16_t* dO_shards, const float* lse, int64_t batch,
                                    int64_t seq, int64_t n_q, int64_t n_kv, int64_t head_dim,
                                    int causal, int n_shards, void* ws, size_t ws_bytes,
                                    uint16_t* dQKV_shards, void* stream) {
  if (QKV_shards == nullptr || O_shards == nullptr || dO_shards == nullptr || lse == nullptr ||
      dQKV_shards == nullptr || ws == nullptr)
    return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || !gqa_ok(n_q, n_kv, n_shards)) return TP_ERR_SHAPE;
  if (head_dim != 128) return TP_ERR_UNSUPPORTED;
  if (batch * seq > kIntMax || seq > kIntMax) return TP_ERR_SHAPE;
  const int64_t M = batch * seq;
  const int64_t hq = n_q * head_dim;  // query columns over all shards
  if (ws_bytes < tp_workspace_bytes(TP_WS_ATTN_CORE_BWD, M, hq, 0, n_shards))
    return TP_ERR_WORKSPACE;
  if (!al16(QKV_shards) || !al16(O_shards) || !al16(dO_shards) || !al16(lse) ||
      !al16(dQKV_shards) || !al16(ws))
    return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  const AttnBwdScratch sc = attn_bwd_scratch(ws, static_cast<size_t>(M), n_q);
  TraceScope ts(tpk::KID_ATTENTION_BWD, as_stream(stream));
  const int rc = tpk::launch_attention_bwd(QKV_shards, O_shards, dO_shards, lse, batch, seq, n_q,
                                           gqa_kv_local(n_kv, n_shards), n_shards,
                                           causal ? 1 : 0, dQKV_shards, sc.dsum, sc.dq_acc,
                                           as_stream(stream), d.err, d.num_sms);
  return rc == 0 ? TP_OK : TP_ERR_CUDA;
}

tp_status tp_attn_backward_gqa(const uint16_t* X, int64_t batch, int64_t seq, int64_t h,
                               int64_t n_q, int64_t n_kv, int causal, int n_shards,
                               const uint16_t* Wqkv_shards, const uint16_t* bqkv_shards,
                               const uint16_t* Wo_shards, const uint16_t* dY, int residual,
                               void* ws, size_t ws_bytes, uint16_t* dX, float* dWqkv_shards,
                               float* dbqkv_shards, float* dWo_shards, float* dbo,
                               void* stream) {
  if (X == nullptr || Wqkv_shards == nullptr || Wo_shards == nullptr || dY == nullptr ||
      dX == nullptr || dWqkv_shards == nullptr || dbqkv_shards == nullptr ||
      dWo_shards == nullptr || dbo == nullptr || ws == nullptr)
    return TP_ERR_NULL;
  if (batch <= 0 || seq <= 0 || h <= 0 || !gqa_ok(n_q, n_kv, n_shards)) return TP_ERR_SHAPE;
  if (h % n_q || h / n_q != 128) return TP_ERR_UNSUPPORTED;
  if (batch * seq > kIntMax || seq > kIntMax) return TP_ERR_SHAPE;
  if (static_cast<int64_t>(n_shards) * batch * (n_q / n_shards) > 65535) return TP_ERR_SHAPE;
  const int64_t M = batch * seq;
  // the attention workspace holds 3h QKV columns, which covers GQA (N <= n_q)
  if (ws_bytes < tp_workspace_bytes(TP_WS_ATTN_BWD, M, h, 0, n_shards)) return TP_ERR_WORKSPACE;
  if (!al16(ws) || !al16(X) || !al16(Wqkv_shards) || !al16(Wo_shards) || !al16(dY) ||
      !al16(dX) || !al16(dWqkv_shards) || !al16(dbqkv_shards) || !al16(dWo_shards) ||
      !al16(dbo) || (bqkv_shards && !al16(bqkv_shards)))
    return TP_ERR_ALIGN;
  DevInfo d;
  tp_status st = device_info(&d);
  if (st != TP_OK) return st;
  const AttnBwdBufs b = attn_bwd_layout(ws, M, h, n_shards);
  const int64_t qkv_cols = n_shards * (n_q / n_shards + 2 * gqa_kv_local(n_kv, n_shards)) * 128;
  // recompute the forward: QKV_i, O_i and the lse
  st = tp_column_linear(X, M, h, Wqkv_shards, bqkv_shards, qkv_cols, n_shards, TP_ACT_NONE,
                        b.qkv, stream);
  if (st != TP_OK) return st;
  st = tp_attention_gqa_lse(b.qkv, batch, seq, n_q, n_kv, 128, causal, n_shards, b.o, b.lse,
                            stream);
  if (st != TP_OK) return st;
  st = attn_backward_core(d, stream, X, batch, seq, h, n_q, n_kv, causal, n_shards, Wqkv_shards,
                          Wo_shards, dY, b, dWqkv_shards, dbqkv_shards, dWo_shards, dbo);
  if (st != TP_OK) return st;
  return tp_reduce_partials(b.part, n_shards, M, h, nullptr, residual ? dY : nullptr, dX, stream);
}
}  // extern "C"
