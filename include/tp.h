/*
 * tp.h - C ABI of libtp.so: the Megatron-LM tensor-parallel Transformer layer
 * on one B200 (sm_100a), with the N tensor-parallel shards held as N
 * independent shard buffers of one GPU.
 *
 * Sources, cited by page title and section:
 *   [TP-LLM] "Tensor Parallelism in Large Language Models: How Megatron-LM
 *            Partitions Multi-Layer Perceptrons and Attention Heads"
 *            (llms.blog): "The Core Primitives: Column-Parallel and
 *            Row-Parallel Linear Layers", "Partitioning the Multi-Layer
 *            Perceptron (MLP) Block", "Partitioning Multi-Head and
 *            Grouped-Query Attention", "Sequence Parallelism".
 *   [M-LM]   "Megatron-LM" (ai360xpert.com), "How It Works".
 *   [INTRO]  "Introduction to Megatron-LM" (apxml.com), "Core Contributions"
 *            (ColumnParallelLinear(in_features, out_features,
 *            tensor_model_parallel_size) example).
 *
 * Conventions shared by every call
 *   - Problem statement of [TP-LLM] "The Core Primitives": X in R^{B x H_in},
 *     W in R^{H_in x H_out}, Y = X W, shard count N. B counts tokens
 *     (batch x sequence).
 *   - Tensors are DEVICE pointers unless a name says host_. bf16 tensors are
 *     passed as uint16_t bit patterns, fp32 as float. Every matrix is
 *     row-major and contiguous. Device pointers must be 16-byte aligned.
 *   - The caller owns every buffer (allocated and freed by the caller); the
 *     library allocates no device memory. Intermediates of the block calls
 *     live in a caller-provided workspace sized by tp_workspace_bytes().
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream). Argument errors are returned before anything is
 *     launched. A device-side failure (a bounded wait that expired inside a
 *     kernel) is recorded in a per-device error word and reported by
 *     tp_get_last_error(); no kernel traps or spins without a bound.
 *   - Weight shards use the packed layout produced by tp_shard_weights():
 *     shard i is stored transposed (K-major), contiguous, one after another.
 *   - Arithmetic: bf16 inputs, fp32 accumulation, bf16 activations between
 *     the kernels, fp32 row-parallel partial sums.
 *   - Per device, the library caches what it looks up once (the device's
 *     error-word address, its SM count, the GEMM's resident CTA count, the
 *     no-alloc array's address), keyed by device ordinal and guarded for
 *     concurrent first calls. They belong to the device's primary context:
 *     after cudaDeviceReset on a device, call nothing of this library on that
 *     device again in the same process.
 */
#ifndef TP_H
#define TP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TP_OK = 0,
    TP_ERR_NULL = 1,        /* a required pointer is NULL */
    TP_ERR_SHAPE = 2,       /* a size <= 0, a dimension not divisible by N
                               (H_out % N, H_in % N, heads % N), or a size
                               not a multiple of 8 elements where stated */
    TP_ERR_ALIGN = 3,       /* a device pointer is not 16-byte aligned */
    TP_ERR_WORKSPACE = 4,   /* ws_bytes < tp_workspace_bytes(...) */
    TP_ERR_UNSUPPORTED = 5, /* an option the kernels do not implement
                               (e.g. head_dim != 128), or not an sm_100 GPU */
    TP_ERR_CUDA = 6,        /* a CUDA runtime or driver call failed */
    TP_ERR_TIMEOUT = 7      /* a bounded wait inside a kernel expired */
} tp_status;

typedef enum {
    /* [TP-LLM] "Column-Parallel Linear Layer": W = [W_1 ... W_N] along
       H_out, W_i in R^{H_in x H_out/N}. Packed shard i = W_i^T, shape
       [H_out/N][H_in]. */
    TP_SPLIT_COLUMN = 0,
    /* [TP-LLM] "Row-Parallel Linear Layer": W = [W_1; ...; W_N] along H_in,
       W_i in R^{H_in/N x H_out}. Packed shard i = W_i^T, shape
       [H_out][H_in/N]. */
    TP_SPLIT_ROW = 1,
    /* [TP-LLM] attention, "Q, K, V Projections": W = [W_Q | W_K | W_V]
       (H_out = 3h), each sliced column-wise by whole heads; shard i owns
       heads [i n_h/N, (i+1) n_h/N), head k being columns [k d, (k+1) d) of
       each projection. Packed shard i = [Q_i | K_i | V_i]^T, shape
       [3h/N][H_in]. */
    TP_SPLIT_QKV_HEADS = 2,
    /* [TP-LLM] MLP block, gated architectures: W = [W_gate | W_up]
       (H_out = 2F), both projections column-parallel. Shard i's columns
       alternate 128 gate features and the same 128 up features (block k =
       gate features [k 128, (k+1) 128) of the shard, then the same up
       features). Packed shard i shape [2F/N][H_in]; F/N % 128 == 0. */
    TP_SPLIT_GATE_UP = 3
} tp_split;

typedef enum {
    TP_ACT_NONE = 0,
    /* GeLU(x) = 0.5 x (1 + erf(x / sqrt 2)), applied per column shard
       ([TP-LLM] "Column-Parallel Linear Layer": an element-wise function is
       applied to the local slice; [M-LM] step 1). */
    TP_ACT_GELU_ERF = 1,
    /* Gated: with TP_SPLIT_GATE_UP weights, Y_i = SiLU(X W_gate,i) *
       (X W_up,i), SiLU(x) = x / (1 + e^-x) ([TP-LLM] MLP block: the gated
       product is local to each shard). Y_shards then has F/N = H_out/(2N)
       columns per shard; no bias. */
    TP_ACT_SWIGLU = 2
} tp_act;

typedef enum {
    TP_WS_MLP = 0, TP_WS_ATTN = 1, TP_WS_LAYER = 2, TP_WS_LAYER_SP = 3, TP_WS_MLP_BWD = 4,
    TP_WS_ATTN_CORE_BWD = 5, TP_WS_ATTN_BWD = 6, TP_WS_LAYER_BWD = 7, TP_WS_LN_BWD = 8,
    TP_WS_LAYER_BWD_SP = 9
} tp_ws_kind;

/* Weights of one pre-LN layer, all device pointers in the packed shard
   layouts below. h = hidden, F = FFN width, N = shards. */
typedef struct {
    const uint16_t* ln1_gamma;   /* [h] */
    const uint16_t* ln1_beta;    /* [h] */
    const uint16_t* Wqkv_shards; /* TP_SPLIT_QKV_HEADS of [h][3h]: [N][3h/N][h] */
    const uint16_t* bqkv_shards; /* TP_SPLIT_QKV_HEADS of [1][3h]: [N][3h/N] */
    const uint16_t* Wo_shards;   /* TP_SPLIT_ROW of [h][h]: [N][h][h/N] */
    const uint16_t* bo;          /* [h], added once after the sum */
    const uint16_t* ln2_gamma;   /* [h] */
    const uint16_t* ln2_beta;    /* [h] */
    const uint16_t* A_shards;    /* TP_SPLIT_COLUMN of [h][F]: [N][F/N][h] */
    const uint16_t* b1_shards;   /* [N][F/N] (= the F-vector b1 itself) */
    const uint16_t* B_shards;    /* TP_SPLIT_ROW of [F][h]: [N][h][F/N] */
    const uint16_t* b2;          /* [h], added once after the sum */
} tp_layer_weights;

/* Gradients of one layer's parameters (fp32 device buffers), in the same
   packed layouts as the weights of tp_layer_weights. */
typedef struct {
    float* ln1_gamma;    /* [h] */
    float* ln1_beta;     /* [h] */
    float* Wqkv_shards;  /* [N][3h/N][h] */
    float* bqkv_shards;  /* [N][3h/N] */
    float* Wo_shards;    /* [N][h][h/N] */
    float* bo;           /* [h] */
    float* ln2_gamma;    /* [h] */
    float* ln2_beta;     /* [h] */
    float* A_shards;     /* [N][F/N][h] */
    float* b1_shards;    /* [N][F/N] */
    float* B_shards;     /* [N][h][F/N] */
    float* b2;           /* [h] */
} tp_layer_grads;

/* tp_shard_weights - pack W (H_in x H_out, bf16) into N shards.
 * [TP-LLM] "The Core Primitives" (column and row splits); attention section
 * (head split). out[i] = W_i^T, contiguous: [N][cols_i][rows_i] with
 * (cols_i, rows_i) = (H_out/N, H_in) for COLUMN, (H_out, H_in/N) for ROW,
 * (H_out/N, H_in) for QKV_HEADS (H_out = 3h, head_dim = d). A bias vector is
 * packed by passing it as a 1 x H_out matrix. Exact copy (bit-for-bit).
 * Errors: TP_ERR_SHAPE if the split dimension is not divisible by N (or, for
 * QKV_HEADS, H_out % 3, h % head_dim or n_heads % N is not 0). W and out
 * must not overlap. */
tp_status tp_shard_weights(const uint16_t* W, int64_t h_in, int64_t h_out,
                           int n_shards, int kind, int64_t head_dim,
                           uint16_t* W_shards, void* stream);

/* tp_shard_index_map - host-only: for every split index (a column of W for
 * COLUMN and QKV_HEADS, a row for ROW) the owning shard and the position
 * inside it. host_owner and host_local are HOST arrays of length H_out
 * (COLUMN, QKV_HEADS) or H_in (ROW). Launches nothing. */
tp_status tp_shard_index_map(int kind, int64_t h_in, int64_t h_out,
                             int n_shards, int64_t head_dim,
                             int32_t* host_owner, int64_t* host_local);

/* tp_column_linear - Y_i = act(X W_i + b_i) for every shard i, one launch.
 * [TP-LLM] "Column-Parallel Linear Layer" (X replicated, Y_i = X W_i, no
 * communication; element-wise activation on the local slice).
 * X [B][H_in]; W_shards [N][H_out/N][H_in] (packed); bias_shards [N][H_out/N]
 * or NULL; Y_shards [N][B][H_out/N] (shard-major: the column gather of
 * [INTRO] is a view, not a copy). H_in and H_out/N must be multiples of 8.
 * With act = TP_ACT_SWIGLU: W_shards is TP_SPLIT_GATE_UP-packed, H_out = 2F
 * counts gate and up columns, (H_out/N) % 256 == 0, bias_shards must be NULL
 * and Y_shards is [N][B][H_out/(2N)]. */
tp_status tp_column_linear(const uint16_t* X, int64_t B, int64_t h_in,
                           const uint16_t* W_shards,
                           const uint16_t* bias_shards, int64_t h_out,
                           int n_shards, int act, uint16_t* Y_shards,
                           void* stream);

/* tp_mlp_forward_swiglu - Y = (SiLU(X W_gate) * (X W_up)) B + b2 + residual
 * by the tensor-parallel route: gate and up column-parallel with the gated
 * product fused into the GEMM epilogue, B row-parallel into N partials, one
 * sum ([TP-LLM] MLP block, gated architectures). X [B][h]; GU_shards
 * TP_SPLIT_GATE_UP of [h][2F]: [N][2F/N][h]; B_shards [N][h][F/N]; b2 [h] or
 * NULL; residual [B][h] or NULL; Y [B][h]. F/N % 128 == 0.
 * ws >= tp_workspace_bytes(TP_WS_MLP, B, h, F, N). */
tp_status tp_mlp_forward_swiglu(const uint16_t* X, int64_t B, int64_t h,
                                int64_t ffn, int n_shards,
                                const uint16_t* GU_shards,
                                const uint16_t* B_shards, const uint16_t* b2,
                                const uint16_t* residual, void* ws,
                                size_t ws_bytes, uint16_t* Y, void* stream);

/* tp_row_linear - partials P_i = X_i W_i (each B x H_out, fp32), one launch.
 * [TP-LLM] "Row-Parallel Linear Layer" (X = [X_1 ... X_N] along channels,
 * Y_i = X_i W_i full size). X_shards [N][B][H_in/N]; W_shards
 * [N][H_out][H_in/N] (packed); partials [N][B][H_out] fp32. H_in/N and H_out
 * must be multiples of 8. */
tp_status tp_row_linear(const uint16_t* X_shards, int64_t B, int64_t h_in,
                        const uint16_t* W_shards, int64_t h_out, int n_shards,
                        float* partials, void* stream);

/* tp_reduce_partials - Y = sum_{i<N} P_i + bias + residual, bf16 out.
 * [TP-LLM] "Row-Parallel Linear Layer" (Y = sum_i Y_i = X W, the all-reduce
 * sum) done as one on-device sum of N shard buffers, fp32 in shard order,
 * one rounding to bf16. partials [N][B][H_out] fp32; bias [H_out] or NULL;
 * residual [B][H_out] or NULL; Y [B][H_out]. H_out % 8 == 0. */
tp_status tp_reduce_partials(const float* partials, int n_shards, int64_t B,
                             int64_t h_out, const uint16_t* bias,
                             const uint16_t* residual, uint16_t* Y,
                             void* stream);

/* tp_reduce_partials_layernorm - the same sum, plus LN of it:
 * S = bf16(sum_i P_i + bias + residual) written to Y_sum, and
 * Y_ln = LN(S) = gamma (S - mean) / sqrt(var + eps) + beta (population
 * variance, fp32 statistics). The residual stream of a pre-LN layer and the
 * next LayerNorm in one pass ([TP-LLM] "Sequence Parallelism": LayerNorm and
 * residual adds are replicated around the blocks). H_out % 8 == 0 and
 * H_out <= 16384. */
tp_status tp_reduce_partials_layernorm(const float* partials, int n_shards,
                                       int64_t B, int64_t h_out,
                                       const uint16_t* bias,
                                       const uint16_t* residual,
                                       const uint16_t* gamma,
                                       const uint16_t* beta, float eps,
                                       uint16_t* Y_sum, uint16_t* Y_ln,
                                       void* stream);

/* tp_layernorm - Y = gamma (X - mean) / sqrt(var + eps) + beta per token row
 * (population variance, fp32 statistics). X, Y [B][h]; gamma, beta [h].
 * h % 8 == 0 and h <= 16384. */
tp_status tp_layernorm(const uint16_t* X, int64_t B, int64_t h,
                       const uint16_t* gamma, const uint16_t* beta, float eps,
                       uint16_t* Y, void* stream);

/* tp_attention - local scaled dot-product attention of every shard's heads:
 * Head = softmax(Q K^T / sqrt(d_k)) V per (sequence, head), d_k = h/n_heads
 * ([TP-LLM] "Local Self-Attention Computation"). With causal != 0 query t
 * of a sequence sees keys 0..t of the same sequence; attention never
 * crosses sequences. QKV_shards [N][batch*seq][3h/N] with each shard's
 * columns [Q_i | K_i | V_i] (the output of tp_column_linear on
 * TP_SPLIT_QKV_HEADS weights); O_shards [N][batch*seq][h/N], the shard's
 * head outputs concatenated in head order. head_dim must be 128. */
tp_status tp_attention(const uint16_t* QKV_shards, int64_t batch,
                       int64_t seq, int64_t h, int64_t n_heads, int causal,
                       int n_shards, uint16_t* O_shards, void* stream);

/* tp_mlp_forward - Y = GeLU(X A + b1) B + b2 + residual, by the
 * tensor-parallel route: column-parallel A with per-shard bias + GeLU,
 * row-parallel B into N fp32 partials, one on-device sum with b2 and the
 * residual ([TP-LLM] "Partitioning the Multi-Layer Perceptron (MLP) Block";
 * [M-LM] "How It Works"). X [B][h]; A_shards [N][F/N][h]; b1_shards [N][F/N]
 * or NULL; B_shards [N][h][F/N]; b2 [h] or NULL; residual [B][h] or NULL;
 * Y [B][h]. ws >= tp_workspace_bytes(TP_WS_MLP, B, h, F, N) bytes. */
tp_status tp_mlp_forward(const uint16_t* X, int64_t B, int64_t h, int64_t ffn,
                         int n_shards, const uint16_t* A_shards,
                         const uint16_t* b1_shards, const uint16_t* B_shards,
                         const uint16_t* b2, const uint16_t* residual,
                         void* ws, size_t ws_bytes, uint16_t* Y, void* stream);

/* tp_mlp_backward - gradients of Y = GeLU(X A + b1) B + b2 (+ X) by the
 * tensor-parallel route ([TP-LLM] MLP block: exactly one all-reduce in the
 * backward pass, of the input gradient across the column-parallel layer).
 * dY reaches every shard whole (the row-parallel layer's backward needs no
 * exchange); each shard recomputes Z_i = X A_i + b1_i (one GEMM whose
 * epilogue emits GeLU(Z_i) and GeLU'(Z_i), both stored as bf16), forms
 * dZ_i = (dY B_i^T) * GeLU'(Z_i), its weight gradients locally, and a
 * full-size partial dX_i = dZ_i A_i^T; dX = sum_i dX_i (+ dY when residual)
 * is the one reduction.
 * Inputs: X [B][h], the forward's packed A_shards [N][F/N][h], b1_shards
 * [N][F/N] or NULL, B_shards [N][h][F/N], dY [B][h] (all bf16).
 * Outputs: dX [B][h] bf16; dA_shards [N][F/N][h] and dB_shards [N][h][F/N]
 * fp32 in the packed layouts of A_shards and B_shards (dA_shards[i] =
 * dA_i^T, dB_shards[i] = dB_i^T); db1 [F] and db2 [h] fp32.
 * ws >= tp_workspace_bytes(TP_WS_MLP_BWD, B, h, F, N). */
tp_status tp_mlp_backward(const uint16_t* X, int64_t B, int64_t h, int64_t ffn,
                          int n_shards, const uint16_t* A_shards,
                          const uint16_t* b1_shards, const uint16_t* B_shards,
                          const uint16_t* dY, int residual, void* ws,
                          size_t ws_bytes, uint16_t* dX, float* dA_shards,
                          float* db1, float* dB_shards, float* db2,
                          void* stream);

/* tp_attention_lse - tp_attention that also writes what its backward needs:
 * for every shard i, local head k and token row r (of batch*seq = M),
 * lse[(i*n_heads/N + k)*(M + 128) + r] = log2 sum_s exp(q_r . k_s / sqrt(d))
 * over the keys s the query sees (the base-2 log-sum-exp of its scaled
 * scores). lse holds n_heads*(M + 128) floats; the last 128 of each head's
 * row are not written. Other arguments as tp_attention. */
tp_status tp_attention_lse(const uint16_t* QKV_shards, int64_t batch,
                           int64_t seq, int64_t h, int64_t n_heads, int causal,
                           int n_shards, uint16_t* O_shards, float* lse,
                           void* stream);

/* tp_attention_backward - gradients of the local attention of every shard's
 * heads (the backward of tp_attention, local to each shard like the forward:
 * [TP-LLM] "Local Self-Attention Computation"). With P = softmax(Q K^T /
 * sqrt d) rebuilt from lse: dV = P^T dO, dP = dO V^T,
 * dS = P * (dP - rowsum(dO * O)), dQ = dS K / sqrt d, dK = dS^T Q / sqrt d.
 * Inputs: QKV_shards [N][M][3h/N], O_shards and dO_shards [N][M][h/N] (bf16)
 * and lse from tp_attention_lse on the same QKV. Output: dQKV_shards
 * [N][M][3h/N] bf16, packed like QKV ([dQ_i | dK_i | dV_i]). Multi-head
 * attention only (no GQA); head_dim must be 128. dQ is accumulated in fp32
 * with atomic additions, so its last bits can differ between runs.
 * ws >= tp_workspace_bytes(TP_WS_ATTN_CORE_BWD, M, h, 0, N). */
tp_status tp_attention_backward(const uint16_t* QKV_shards,
                                const uint16_t* O_shards,
                                const uint16_t* dO_shards, const float* lse,
                                int64_t batch, int64_t seq, int64_t h,
                                int64_t n_heads, int causal, int n_shards,
                                void* ws, size_t ws_bytes,
                                uint16_t* dQKV_shards, void* stream);

/* tp_attn_backward - gradients of the attention block
 * Y = concat_heads(attention) W_O + b_O (+ X) by the tensor-parallel route:
 * dY reaches every shard whole (the row-parallel W_O's backward needs no
 * exchange); shard i recomputes QKV_i, O_i and lse, forms dO_i = dY W_O,i^T,
 * its heads' attention backward, its weight gradients locally and a
 * full-size partial dX_i = dQKV_i W_QKV,i^T; dX = sum_i dX_i (+ dY when
 * residual) is the block's one reduction ([TP-LLM] "Communication Budget and
 * Scaling Limits": two all-reduces per layer in the backward pass, one per
 * block). Inputs as tp_attn_forward plus dY [M][h] (bf16). Outputs: dX [M][h]
 * bf16; dWqkv_shards [N][3h/N][h], dbqkv_shards [N][3h/N], dWo_shards
 * [N][h][h/N] fp32 in the packed layouts of the weights; dbo [h] fp32.
 * ws >= tp_workspace_bytes(TP_WS_ATTN_BWD, M, h, 0, N). */
tp_status tp_attn_backward(const uint16_t* X, int64_t batch, int64_t seq,
                           int64_t h, int64_t n_heads, int causal, int n_shards,
                           const uint16_t* Wqkv_shards,
                           const uint16_t* bqkv_shards,
                           const uint16_t* Wo_shards, const uint16_t* dY,
                           int residual, void* ws, size_t ws_bytes,
                           uint16_t* dX, float* dWqkv_shards,
                           float* dbqkv_shards, float* dWo_shards, float* dbo,
                           void* stream);

/* tp_reduce_partials_layernorm_backward - the backward reduction of a pre-LN
 * block: g = sum_i partials_i (the gradient reaching LN(x), the block's one
 * reduction, fp32 sum in shard order) through the LayerNorm backward, plus the
 * residual gradient:
 *   dX = residual_grad + rstd (g gamma - mean(g gamma) - x_hat mean(g gamma x_hat))
 * per row (x_hat = (x - mean) rstd, population variance, eps as the forward),
 * dgamma = sum_rows g x_hat, dbeta = sum_rows g (fp32, deterministic).
 * partials [N][B][h] fp32; x (the LN input), residual_grad (or NULL), dX
 * [B][h] bf16; gamma [h] bf16. h % 8 == 0, h <= 16384.
 * ws >= tp_workspace_bytes(TP_WS_LN_BWD, B, h, 0, N). */
tp_status tp_reduce_partials_layernorm_backward(const float* partials, int n_shards,
                                                int64_t B, int64_t h, const uint16_t* x,
                                                const uint16_t* gamma,
                                                const uint16_t* residual_grad, float eps,
                                                void* ws, size_t ws_bytes, uint16_t* dX,
                                                float* dgamma, float* dbeta, void* stream);

/* tp_layer_backward - gradients of the pre-LN layer of tp_layer_forward
 * (causal attention) by the tensor-parallel route: the forward is recomputed
 * from X (LN1, QKV, attention with its log-sum-exp, W_O, LN2); the MLP
 * block's backward ends in its one reduction, fused with LN2's backward and
 * the residual (dh1 = dY + LN2'^T sum_i dx2_i); the attention block's backward
 * ends in its one reduction, fused with LN1's backward and the residual
 * (dX = dh1 + LN1'^T sum_i dx1_i): two reductions in the backward pass, as
 * [TP-LLM] "Communication Budget and Scaling Limits" counts. X, dY, dX
 * [batch*seq][h] bf16; w as tp_layer_forward; g receives every parameter
 * gradient (fp32, packed layouts). head_dim must be 128.
 * ws >= tp_workspace_bytes(TP_WS_LAYER_BWD, batch*seq, h, F, N). */
tp_status tp_layer_backward(const uint16_t* X, int64_t batch, int64_t seq,
                            int64_t h, int64_t n_heads, int64_t ffn,
                            int n_shards, const tp_layer_weights* w,
                            float ln_eps, const uint16_t* dY, void* ws,
                            size_t ws_bytes, uint16_t* dX,
                            const tp_layer_grads* g, void* stream);

/* tp_attention_gqa_lse - tp_attention_gqa that also writes the base-2
 * log-sum-exp of every query's scaled scores, laid out as in
 * tp_attention_lse (n_q*(batch*seq + 128) floats, query heads in shard
 * order). */
tp_status tp_attention_gqa_lse(const uint16_t* QKV_shards, int64_t batch,
                               int64_t seq, int64_t n_q, int64_t n_kv,
                               int64_t head_dim, int causal, int n_shards,
                               uint16_t* O_shards, float* lse, void* stream);

/* tp_attention_gqa_backward - tp_attention_backward for grouped-query QKV
 * shards (the layout of tp_shard_qkv_gqa): a key/value head's dK and dV are
 * summed over the local query heads of its group ([TP-LLM] "Grouped-Query
 * Attention (GQA) Constraints"). When N > n_kv each shard's duplicated
 * key/value head receives the gradient of that shard's query heads only; the
 * gradient of the logical head is the sum over its replicas. dQKV_shards is
 * packed like QKV_shards. ws >= tp_workspace_bytes(TP_WS_ATTN_CORE_BWD, M,
 * n_q*head_dim, 0, N). */
tp_status tp_attention_gqa_backward(const uint16_t* QKV_shards,
                                    const uint16_t* O_shards,
                                    const uint16_t* dO_shards, const float* lse,
                                    int64_t batch, int64_t seq, int64_t n_q,
                                    int64_t n_kv, int64_t head_dim, int causal,
                                    int n_shards, void* ws, size_t ws_bytes,
                                    uint16_t* dQKV_shards, void* stream);

/* tp_attn_backward_gqa - tp_attn_backward for the grouped-query block of
 * tp_attn_forward_gqa (h = n_q * 128). dWqkv_shards and dbqkv_shards are
 * packed like the GQA shards ([N][(n_q/N + 2 kv_local) 128][h] and
 * [N][(n_q/N + 2 kv_local) 128]); a duplicated key/value head's columns hold
 * that shard's share of its gradient. ws >= tp_workspace_bytes(TP_WS_ATTN_BWD,
 * M, h, 0, N). */
tp_status tp_attn_backward_gqa(const uint16_t* X, int64_t batch, int64_t seq,
                               int64_t h, int64_t n_q, int64_t n_kv, int causal,
                               int n_shards, const uint16_t* Wqkv_shards,
                               const uint16_t* bqkv_shards,
                               const uint16_t* Wo_shards, const uint16_t* dY,
                               int residual, void* ws, size_t ws_bytes,
                               uint16_t* dX, float* dWqkv_shards,
                               float* dbqkv_shards, float* dWo_shards,
                               float* dbo, void* stream);

/* tp_layer_backward_sp - tp_layer_backward under sequence parallelism: X,
 * dY and dX in the sequence-sharded layout [N][batch][seq/N][h] of
 * tp_layer_forward_sp ([TP-LLM] "Sequence Parallelism"). The backward swaps
 * the forward's collectives: dY and dh1 are all-gathered before each block,
 * and each block's one reduction is a reduce-scatter fused with the LN
 * backward and the residual. Gradients as tp_layer_backward.
 * ws >= tp_workspace_bytes(TP_WS_LAYER_BWD_SP, batch*seq, h, F, N). */
tp_status tp_layer_backward_sp(const uint16_t* X_shards, int64_t batch,
                               int64_t seq, int64_t h, int64_t n_heads,
                               int64_t ffn, int n_shards,
                               const tp_layer_weights* w, float ln_eps,
                               const uint16_t* dY_shards, void* ws,
                               size_t ws_bytes, uint16_t* dX_shards,
                               const tp_layer_grads* g, void* stream);

/* tp_attn_forward - Y = concat_heads(attention) W_O + b_O + residual by the
 * tensor-parallel route: QKV column-parallel by whole heads (+ bias), local
 * attention per shard, W_O row-parallel into N partials, one sum
 * ([TP-LLM] "Partitioning Multi-Head and Grouped-Query Attention" steps
 * 1-4). X [batch*seq][h]; Wqkv_shards [N][3h/N][h]; bqkv_shards [N][3h/N] or
 * NULL; Wo_shards [N][h][h/N]; bo [h] or NULL; residual [batch*seq][h] or
 * NULL; Y [batch*seq][h]. head_dim = h/n_heads must be 128.
 * ws >= tp_workspace_bytes(TP_WS_ATTN, batch*seq, h, 0, N). */
tp_status tp_attn_forward(const uint16_t* X, int64_t batch, int64_t seq,
                          int64_t h, int64_t n_heads, int causal,
                          int n_shards, const uint16_t* Wqkv_shards,
                          const uint16_t* bqkv_shards,
                          const uint16_t* Wo_shards, const uint16_t* bo,
                          const uint16_t* residual, void* ws, size_t ws_bytes,
                          uint16_t* Y, void* stream);

/* tp_layer_forward - pre-LN Transformer layer, causal attention:
 * h1 = X + Attn(LN1(X)); Y = h1 + MLP(LN2(h1)), both blocks by the
 * tensor-parallel route with one partial-sum reduction each.
 * X, Y [batch*seq][h]; w: see tp_layer_weights.
 * ws >= tp_workspace_bytes(TP_WS_LAYER, batch*seq, h, F, N). */
tp_status tp_layer_forward(const uint16_t* X, int64_t batch, int64_t seq,
                           int64_t h, int64_t n_heads, int64_t ffn,
                           int n_shards, const tp_layer_weights* w,
                           float ln_eps, void* ws, size_t ws_bytes,
                           uint16_t* Y, void* stream);

/* ---- Grouped-query attention ([TP-LLM] "Grouped-Query Attention (GQA)
 * Constraints") ------------------------------------------------------------
 * W_QKV = [W_Q | W_K | W_V] with n_q query heads and n_kv key/value heads of
 * head_dim d (W_Q h x n_q d; W_K, W_V h x n_kv d); query head j uses kv head
 * j / (n_q / n_kv). Requires n_q % N == 0, n_q % n_kv == 0 and either
 * n_kv % N == 0 (shard i owns n_kv/N whole groups) or N % n_kv == 0 (N >
 * n_kv: each shard holds a duplicate of its group's kv head). Shard i's
 * columns: [Q_i (n_q/N heads) | K_i | V_i (kv_local heads each)], kv_local =
 * n_kv/N or 1. Errors: TP_ERR_SHAPE for any other (n_q, n_kv, N). */

/* Pack W_QKV [h_in][(n_q + 2 n_kv) d] into [N][(n_q/N + 2 kv_local) d][h_in]
 * (a bias is packed as a 1-row matrix). Exact copy. */
tp_status tp_shard_qkv_gqa(const uint16_t* W, int64_t h_in, int64_t n_q,
                           int64_t n_kv, int64_t head_dim, int n_shards,
                           uint16_t* W_shards, void* stream);

/* Local attention of every shard's query heads with their group's kv head.
 * QKV_shards [N][batch*seq][(n_q/N + 2 kv_local) d]; O_shards
 * [N][batch*seq][n_q d / N]. head_dim must be 128. */
tp_status tp_attention_gqa(const uint16_t* QKV_shards, int64_t batch,
                           int64_t seq, int64_t n_q, int64_t n_kv,
                           int64_t head_dim, int causal, int n_shards,
                           uint16_t* O_shards, void* stream);

/* GQA attention block by the tensor-parallel route (h = n_q x 128):
 * Wqkv_shards from tp_shard_qkv_gqa, bqkv_shards likewise or NULL,
 * Wo_shards TP_SPLIT_ROW of [h][h], bo [h] or NULL, residual [M][h] or NULL.
 * ws >= tp_workspace_bytes(TP_WS_ATTN, batch*seq, h, 0, N). */
tp_status tp_attn_forward_gqa(const uint16_t* X, int64_t batch, int64_t seq,
                              int64_t h, int64_t n_q, int64_t n_kv, int causal,
                              int n_shards, const uint16_t* Wqkv_shards,
                              const uint16_t* bqkv_shards,
                              const uint16_t* Wo_shards, const uint16_t* bo,
                              const uint16_t* residual, void* ws,
                              size_t ws_bytes, uint16_t* Y, void* stream);

/* ---- Sequence parallelism ([TP-LLM] "Sequence Parallelism") ----------
 * Outside the tensor-parallel blocks, activations are split along the
 * sequence: shard i owns positions [i S/N, (i+1) S/N) of every sequence.
 * Sequence-sharded layout: [N][batch][S/N][h], i.e. token (b, s) of a
 * token-ordered [batch*S][h] tensor lives at
 * [s / (S/N)][b][s % (S/N)][:]. seq % N must be 0. */

/* tp_reduce_scatter_partials - the reduce-scatter after a row-parallel layer:
 * Y_shards (sequence-sharded) = slices of (sum_{i<N} P_i + bias), plus the
 * residual given in the same sharded layout (NULL ok). partials
 * [N][batch*seq][h] fp32 in token order; bias [h] or NULL. An all-reduce is
 * this followed by tp_all_gather_sequence. h % 8 == 0. */
tp_status tp_reduce_scatter_partials(const float* partials, int n_shards,
                                     int64_t batch, int64_t seq, int64_t h,
                                     const uint16_t* bias,
                                     const uint16_t* residual_shards,
                                     uint16_t* Y_shards, void* stream);

/* tp_all_gather_sequence - the all-gather before a column-parallel layer:
 * X [batch*seq][h] (token order) from X_shards (sequence-sharded). A pure
 * permutation copy. h % 8 == 0. */
tp_status tp_all_gather_sequence(const uint16_t* X_shards, int n_shards,
                                 int64_t batch, int64_t seq, int64_t h,
                                 uint16_t* X, void* stream);

/* tp_layer_forward_sp - the pre-LN layer of tp_layer_forward with sequence
 * parallelism: X_shards and Y_shards in the sequence-sharded layout;
 * LayerNorm on each shard's slice followed by the all-gather (one fused
 * kernel), reduce-scatter after each row-parallel layer (fused with the
 * bias, the sharded residual and, after attention, LN2 + all-gather).
 * Same result as tp_layer_forward up to the row order.
 * ws >= tp_workspace_bytes(TP_WS_LAYER_SP, batch*seq, h, F, N). */
tp_status tp_layer_forward_sp(const uint16_t* X_shards, int64_t batch,
                              int64_t seq, int64_t h, int64_t n_heads,
                              int64_t ffn, int n_shards,
                              const tp_layer_weights* w, float ln_eps,
                              void* ws, size_t ws_bytes, uint16_t* Y_shards,
                              void* stream);

/* Size in bytes of the library-owned scratch array used by
 * tp_mlp_forward_noalloc (32 MiB per GPU). The array belongs to the CUDA
 * module of the file that defines it; the CUDA runtime reserves it on a GPU
 * when it loads that module there. With lazy module loading (the CUDA 12
 * default, CUDA_MODULE_LOADING=LAZY) that is the first
 * tp_mlp_forward_noalloc call on that GPU; with eager loading it is the
 * first CUDA call of the process that creates the GPU's context. It stays
 * reserved until the process exits. */
#define TP_NOALLOC_WS_BYTES (32u * 1024u * 1024u)

/* tp_mlp_forward_noalloc - tp_mlp_forward for callers that cannot allocate
 * device memory: the same arguments and result, but without the workspace
 * pair; the intermediates live in a fixed library-owned device array of
 * TP_NOALLOC_WS_BYTES. The pages have no counterpart to this call: it exists
 * for callers that have no device allocator to hand (a C program embedding
 * the library without a memory pool) or whose framework has already reserved
 * all device memory, so they cannot ask for a workspace.
 * - Rejects, with TP_ERR_WORKSPACE and before any launch, a problem whose
 *   tp_workspace_bytes(TP_WS_MLP, B, h, ffn, N) exceeds TP_NOALLOC_WS_BYTES.
 * - All calls on a device share the array; it keeps the last call's contents
 *   (no part of it needs to start at zero). Calls that overlap on the GPU
 *   (unordered streams or host threads) race on it: the caller must order
 *   them.
 * - The first call on a device looks up and caches the array's device
 *   address (cudaGetSymbolAddress, with that device current). Under lazy
 *   module loading that lookup is also what loads the module and reserves
 *   the 32 MiB, so a caller whose memory pool later takes all free device
 *   memory must make its first call BEFORE the pool reserves it, and before
 *   any stream capture begins. If the GPU has no room left for the array at
 *   that point the call returns TP_ERR_WORKSPACE (nothing is launched).
 * - The cached address is that of the device's primary context: after
 *   cudaDeviceReset on a device, call nothing of this library on it again in
 *   the same process.
 * - Calls no cudaMalloc, cudaFree or other allocating routine itself. */
tp_status tp_mlp_forward_noalloc(const uint16_t* X, int64_t B, int64_t h,
                                 int64_t ffn, int n_shards,
                                 const uint16_t* A_shards,
                                 const uint16_t* b1_shards,
                                 const uint16_t* B_shards, const uint16_t* b2,
                                 const uint16_t* residual, uint16_t* Y,
                                 void* stream);

/* Workspace bytes for tp_mlp_forward (kind TP_WS_MLP), tp_attn_forward
 * (TP_WS_ATTN, ffn ignored), tp_layer_forward (TP_WS_LAYER),
 * tp_layer_forward_sp (TP_WS_LAYER_SP), tp_mlp_backward (TP_WS_MLP_BWD),
 * tp_attention_backward (TP_WS_ATTN_CORE_BWD, ffn ignored), tp_attn_backward
 * (TP_WS_ATTN_BWD, ffn ignored), tp_layer_backward (TP_WS_LAYER_BWD),
 * tp_layer_backward_sp (TP_WS_LAYER_BWD_SP) or
 * tp_reduce_partials_layernorm_backward (TP_WS_LN_BWD, tokens and ffn ignored).
 * tokens = batch * seq. Returns 0 for invalid arguments. */
size_t tp_workspace_bytes(int kind, int64_t tokens, int64_t h, int64_t ffn,
                          int n_shards);

/* Synchronizes `stream`, then reads and clears the current device's error
 * word. TP_ERR_TIMEOUT if a kernel gave up a bounded wait since the last
 * call, TP_ERR_CUDA if the stream reports a CUDA error, else TP_OK. */
tp_status tp_get_last_error(void* stream);

/* tp_selftest_wait_timeout - a self-test of the failure path, with no
 * counterpart on the pages: launches, on `stream`, one thread that waits for
 * at most limit_us microseconds (1 .. 1000000) on an mbarrier that nothing
 * arrives on, then gives up the way every bounded wait in the library does
 * (a bit in the device's error word). The next tp_get_last_error returns
 * TP_ERR_TIMEOUT and clears the word; the context stays usable. Returns
 * TP_ERR_SHAPE for a limit out of range, TP_ERR_CUDA if the launch fails. */
tp_status tp_selftest_wait_timeout(int64_t limit_us, void* stream);

/* Static string for a status code. */
const char* tp_status_string(int status);

/* Kernel launch trace (used by benchmarks): while enabled, every kernel the
 * library launches is bracketed by two CUDA events on its stream.
 * tp_trace_begin(max_records) starts a trace (max_records launches at most;
 * later launches are counted but not timed); tp_trace_end() synchronizes
 * the device and returns the number of launches seen. tp_trace_record(k)
 * gives launch k's kernel id (host_kernel_id) and its device time in
 * milliseconds (host_ms). Kernel ids are those of tp_kernel_name(). */
tp_status tp_trace_begin(int max_records);
int tp_trace_end(void);
tp_status tp_trace_record(int k, int* host_kernel_id, float* host_ms);
const char* tp_kernel_name(int kernel_id);

#ifdef __cplusplus
}
#endif
#endif /* TP_H */
