/*
 * qg.h -- C ABI of libqg, weight-only-quantized decode kernels for NVIDIA
 * B200 (sm_100a).
 *
 * Sources the operations follow (cited per entry point):
 *   [TS] turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs: resident packed
 *        affine-INT8 (group 64) Qwen3 text decoder (`PackedLinear`,
 *        `load_packed_linear`, `embed_row_bytes`, `step`, `argmax`).
 *   [FT] fuel-transformers 0.19.1, src/models/lazy_quantized_whisper.rs:
 *        GGUF Q4_0 Whisper (`quantize_in_out_to_q4_0`, `q_linear`,
 *        `encoder_layer`).
 *   [MK] makima commit eabd130, src/tts/qwen3/model.rs: candle Qwen3
 *        decoder (`RotaryEmbedding`, `Qwen3Attention::forward`, `repeat_kv`,
 *        `Qwen3Mlp::forward`).
 *
 * Conventions (every entry point):
 *   - Returns a qg_status. On failure qg_last_error() gives a message that
 *     names the offending argument. A call that fails validation launches
 *     nothing and writes nothing.
 *   - Pointers documented as "device" must point to device memory of the
 *     current CUDA device. The library borrows them for the call; it never
 *     allocates, frees or retains them. The caller owns all memory,
 *     workspace included.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream). Results are valid once the stream has
 *     been synchronised. No entry point synchronises, allocates, or
 *     branches on device data on the host, so every compute entry point may
 *     be captured into a CUDA graph.
 *   - Dimensions are int and must be >= 0; an element count that overflows
 *     int64 or a shape rule below is refused with QG_ERR_UNSUPPORTED_SHAPE.
 *     A zero batch or zero row count is a valid no-op.
 *   - bf16 values travel as uint16_t bit patterns.
 *   - Every device pointer must be 16-byte aligned unless stated otherwise
 *     (QG_ERR_MISALIGNED).
 *   - A CUDA launch error returns QG_ERR_CUDA with the CUDA error string.
 */
#ifndef QG_H
#define QG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qg_status {
  QG_OK = 0,
  QG_ERR_INVALID_ARGUMENT = 1,
  QG_ERR_UNSUPPORTED_SHAPE = 2,
  QG_ERR_MISALIGNED = 3,
  QG_ERR_WORKSPACE_TOO_SMALL = 4,
  QG_ERR_CUDA = 5,
  QG_ERR_TIMEOUT = 6
} qg_status;

typedef enum qg_dtype { QG_F32 = 0, QG_BF16 = 1 } qg_dtype;

/* Thread-local message for the last failing call on this host thread
 * ("" after a successful call). Never NULL. */
const char* qg_last_error(void);

/* Version of this ABI (incremented on any incompatible change). */
int qg_abi_version(void);

/* Number of CUDA kernels this library has enqueued in this process (all
 * entry points, all host threads). Capturing a call into a CUDA graph and
 * reading the count before and after gives the kernels per graph replay;
 * a replay of a recorded step graph (qg_decode_step) adds nothing. */
unsigned long long qg_kernel_launch_count(void);

/* ------------------------------------------------------------------------
 * Affine-INT8 group-64 dequant GEMV  [TS: PackedLinear / load_packed_linear,
 * the per-linear GEMV of `step`]
 *
 *   y[b][r] = sum_c (q[r][c] * s[r][c/64] + beta[r][c/64]) * x[b][c]
 *             (+ residual[b][r] when residual != NULL)
 *
 * w       device, uint32 [N][K/4]: row r holds the K code bytes of row r,
 *         column 4j+i in byte i (bits 8i..8i+7) of word j (little endian).
 * scales  device, bf16 [N][K/64] (2-byte alignment suffices).
 * biases  device, bf16 [N][K/64] (2-byte alignment suffices).
 * x       device, [B][K] of x_dtype (QG_BF16 or QG_F32).
 * y       device, [B][N] of y_dtype; fp32 accumulation, one rounding at the
 *         store when y_dtype is QG_BF16. May alias `residual` (in-place
 *         y += W x); must not overlap w, scales, biases or x.
 * residual device fp32 [B][N] or NULL (4-byte alignment suffices).
 * Shape rules: K % 64 == 0, 1 <= B <= 32 (B == 0 is a no-op), N >= 0.
 * Launch: with Programmatic Dependent Launch, so a chain of calls overlaps
 * each GEMV's first weight loads with the previous kernel's tail; the kernel
 * waits for the stream's previous kernel before it reads x or residual.
 * w, scales and biases must not be written by the kernel just before the
 * call on the stream (the first weight loads are issued before that wait).
 * With bf16 x, B >= 5 and a matrix of at least one 128-row tile per SM (the
 * LM head), the call runs qg_gemm_affine8_g64's tensor-core matmul kernel
 * instead (same results within the tolerance; its bounded device-side
 * waits report nothing through this entry point).
 * ---------------------------------------------------------------------- */
qg_status qg_gemv_affine8_g64(const uint32_t* w, const uint16_t* scales,
                              const uint16_t* biases, const void* x,
                              qg_dtype x_dtype, void* y, qg_dtype y_dtype,
                              const float* residual, int N, int K, int B,
                              void* stream);

/* ------------------------------------------------------------------------
 * Q4_0 dequant GEMV  [FT: quantize_in_out_to_q4_0 (block layout), q_linear]
 *
 *   y[b][r] = sum_blk d[r][blk] * sum_{j<32} (n[r][blk][j] - 8) * x[b][32 blk + j]
 *             (+ bias[r] when bias != NULL)
 *
 * blocks  device, uint8 [N][(K/32) * 18]: per block an fp16 d (little
 *         endian) then 16 bytes; byte j holds code j (low nibble) and code
 *         j+16 (high nibble). Rows are contiguous; no padding. 2-byte
 *         alignment suffices.
 * x       device fp32 [B][K].   bias device fp32 [N] or NULL (4-byte align).
 * y       device fp32 [B][N].
 * Shape rules: K % 32 == 0, 1 <= B <= 32 (B == 0 is a no-op).
 * Launch: with Programmatic Dependent Launch (as qg_gemv_affine8_g64); the
 * kernel waits for the stream's previous kernel before it reads x or bias.
 * ---------------------------------------------------------------------- */
qg_status qg_gemv_q4_0(const uint8_t* blocks, const float* x, const float* bias,
                       float* y, int N, int K, int B, void* stream);

/* ------------------------------------------------------------------------
 * Q4_0 matmul on the tensor cores  [FT: encoder_layer -> q_linear with
 * M = frames]
 *
 *   C[m][r] = sum_k bf16(A[m][k]) * bf16(d * (n - 8))[r][k] (+ bias[r])
 *
 * Operands are rounded to bf16 (nearest even) and multiplied on the
 * tcgen05 tensor cores with fp32 accumulation in tensor memory.
 * blocks  device, Q4_0 [N][(K/32)*18] as in qg_gemv_q4_0.
 * A       device fp32 [M][K].  bias device fp32 [N] or NULL.  C device fp32 [M][N].
 * ws      device workspace of at least qg_gemm_q4_0_workspace_size(M,N,K)
 *         bytes, 256-byte aligned (contents need not be initialised): A as
 *         bf16, then the error word.
 * A and C must be 16-byte aligned, blocks 2-byte aligned.
 * Shape rules: K % 64 == 0, N % 128 == 0, M >= 0.
 * ---------------------------------------------------------------------- */
size_t qg_gemm_q4_0_workspace_size(int M, int N, int K);
qg_status qg_gemm_q4_0(const uint8_t* blocks, const float* A, const float* bias,
                       float* C, int M, int N, int K, void* ws, size_t ws_bytes,
                       void* stream);
/* Reads the device error word of the last qg_gemm_q4_0 call that used `ws`
 * (synchronises `stream`). Every device-side wait in the GEMM is bounded
 * (1 s); one that gives up leaves C undefined, records a nonzero code, and
 * this call then returns QG_ERR_TIMEOUT with the code in *code. After a
 * qg_gemm_q4_0_ex call with a bf16 A, pass M = K = 0 (the word then heads
 * the workspace). */
qg_status qg_gemm_q4_0_error(int M, int K, const void* ws, unsigned* code, void* stream);

/* Test aid for the timeout path (no counterpart on the pages): runs the
 * matmul's kernel (bf16 A [M][K]) with every load withheld and no producer
 * arriving, so its MMA issuer's first bounded wait runs out after about
 * 1 ms while nothing is in flight; the kernel then frees its tensor memory
 * and records a nonzero error word in ws (256 bytes, 256-byte aligned),
 * which qg_gemm_q4_0_error(0, 0, ws, ...) reports as QG_ERR_TIMEOUT. C is
 * not written. */
qg_status qg_gemm_q4_0_stall_test(const uint8_t* blocks, const uint16_t* A, float* C, int M,
                                  int N, int K, void* ws, size_t ws_bytes, void* stream);

/* The same matmul with the operand and epilogue options the Whisper encoder
 * layer needs  [FT: encoder_layer -> q_linear, gelu_tanh, residual adds]:
 *
 *   v = sum_k bf16(A[m][k]) * bf16(d * (n - 8))[r][k] + bias[r]
 *       (+ residual[m][r]);   v = gelu_tanh(v) when gelu != 0;
 *   C[m][r] = v as fp32, or rounded to bf16 (nearest even).
 *
 * gelu_tanh(v) = 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))), in fp32.
 * A        device [M][K] of a_dtype: QG_BF16 is read as is (no conversion
 *          pass), QG_F32 is rounded into the workspace first.
 * bias     device fp32 [N] or NULL.  residual device fp32 [M][N] or NULL
 *          (only with c_dtype QG_F32; C may alias it).
 * C        device [M][N] of c_dtype.
 * ws       >= 256 bytes with a bf16 A (the error word), else
 *          qg_gemm_q4_0_workspace_size(M, N, K); 256-byte aligned.
 * A, C and residual 16-byte aligned; shape rules as qg_gemm_q4_0. */
qg_status qg_gemm_q4_0_ex(const uint8_t* blocks, const void* A, qg_dtype a_dtype,
                          const float* bias, const float* residual, void* C, qg_dtype c_dtype,
                          int gelu, int M, int N, int K, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * RMSNorm  [TS: encode_rms_norm_bf16w in `step`; MK: rms_norm layers]
 *   y[r][i] = x[r][i] / sqrt(mean_i(x[r][i]^2) + eps) * w[i]
 * x device fp32 [rows][dim]; w device bf16 [dim] (2-byte alignment);
 * y device [rows][dim] of y_dtype (may alias x when y_dtype is QG_F32).
 * Shape rules: 1 <= dim <= 65536, dim % 4 == 0.
 * ---------------------------------------------------------------------- */
qg_status qg_rmsnorm(const float* x, const uint16_t* w, float eps, void* y,
                     qg_dtype y_dtype, int rows, int dim, void* stream);

/* Per-head RMSNorm (Qwen3 q_norm / k_norm)  [TS: encode_rms_norm_bf16w_perhead;
 * MK: apply_head_norm]: the RMSNorm above on every D-wide slice of
 * x [rows][heads*D] with one shared weight w [D]. x and y fp32 or bf16
 * (x_dtype, y_dtype); y may alias x when the dtypes match.
 * Shape rules: D % 32 == 0, D <= 1024. */
qg_status qg_rmsnorm_perhead(const void* x, qg_dtype x_dtype, const uint16_t* w,
                             float eps, void* y, qg_dtype y_dtype, int rows,
                             int heads, int D, void* stream);

/* ------------------------------------------------------------------------
 * NeoX rotate-half RoPE, in place  [MK: RotaryEmbedding::new / apply /
 * rotate_half; TS: encode_rope_neox_subdim]
 *   for i < rotary_dim/2, a = pos[r] * theta^(-2i/rotary_dim) (float64):
 *   x'[i]      = x[i] cos a - x[i+half] sin a
 *   x'[i+half] = x[i+half] cos a + x[i] sin a,   half = rotary_dim/2;
 *   dims >= rotary_dim are untouched.
 * x device [rows][heads*D] of dtype; pos device int32 [rows] (4-byte align).
 * Shape rules: rotary_dim even, 2 <= rotary_dim <= D, D % 2 == 0.
 * ---------------------------------------------------------------------- */
qg_status qg_rope_neox(void* x, qg_dtype dtype, const int32_t* pos, double theta,
                       int rows, int heads, int D, int rotary_dim, void* stream);

/* SiLU-mul  [TS: encode_silu_mul; MK: Qwen3Mlp::forward]
 *   out[i] = gate[i] / (1 + exp(-gate[i])) * up[i]
 * gate, up device fp32 [n]; out device [n] of out_dtype (may alias gate
 * when QG_F32). 4-byte alignment suffices. */
qg_status qg_silu_mul(const float* gate, const float* up, void* out,
                      qg_dtype out_dtype, int n, void* stream);

/* Residual add  [TS: encode_residual_add]: x[i] += delta[i], fp32, device,
 * 4-byte alignment suffices. */
qg_status qg_residual_add(float* x, const float* delta, int n, void* stream);

/* Tied-embedding row dequantization  [TS: embed_row_bytes]
 *   x[b][c] = q_E[t_b][c] * s_E[t_b][c/64] + beta_E[t_b][c/64]   (fp32)
 * table as in qg_gemv_affine8_g64 with N = vocab, K = hidden; tokens
 * device int32 [B]. A token outside [0, vocab) yields a row of NaN.
 * Shape rules: hidden % 64 == 0. */
qg_status qg_embed_affine8_g64(const uint32_t* w, const uint16_t* scales,
                               const uint16_t* biases, const int32_t* tokens,
                               float* x, int vocab, int hidden, int B,
                               void* stream);

/* ------------------------------------------------------------------------
 * Split-softmax GQA decode attention  [TS: encode_attention_decode with
 * kv_start = 0 and its AttentionScratch; MK: Qwen3Attention::forward,
 * repeat_kv]
 *   For sequence b and query head h (KV head h / (H/Hkv)), L = kv_len[b]:
 *   out[b][h] = sum_{t<L} softmax_t(q[b][h] . k[b][kv][t] * scale) v[b][kv][t]
 * The L rows are cut into chunks scored by separate CTAs; per-chunk
 * (max, sum, weighted V) partials are merged in a fixed order (results do
 * not depend on scheduling). For head_dim 32, 64, 128 or 256 with at most 4
 * query heads per KV head, the chunks of one (sequence, KV head) form a
 * thread-block cluster and merge through distributed shared memory (the
 * workspace is then not touched); other shapes merge through the
 * workspace.
 * q        device fp32 [B][H][D].
 * k_cache, v_cache device bf16 [B][Hkv][cap][D] (row t of head kv at
 *          ((b*Hkv + kv)*cap + t)*D).
 * kv_len   device int32 [B]; read on the device. A value outside [1, cap]
 *          gives a zero output row for that sequence (nothing is read out
 *          of bounds).
 * out      device [B][H][D] of out_dtype.
 * ws       device workspace, >= qg_decode_attention_workspace_size(...)
 *          bytes, 256-byte aligned; its contents need not be initialised.
 * Shape rules: H % Hkv == 0, H/Hkv <= 8, D % 32 == 0, D <= 256, cap >= 1.
 * ---------------------------------------------------------------------- */
size_t qg_decode_attention_workspace_size(int B, int H, int Hkv, int D, int cap);
qg_status qg_decode_attention(const float* q, const uint16_t* k_cache,
                              const uint16_t* v_cache, const int32_t* kv_len,
                              void* out, qg_dtype out_dtype, int B, int H,
                              int Hkv, int D, int cap, float scale, void* ws,
                              size_t ws_bytes, void* stream);

/* qg_decode_attention without a caller workspace. The pages have no
 * counterpart: this is a library convenience, not a step of the method.
 *
 * Who needs it: callers that cannot hand the library device memory at the
 * point of the call -- a plain C host that holds only the cache and
 * activation buffers and has no device allocator, or a decode loop that
 * must not call cudaMalloc / cudaFree between steps (cudaFree synchronises
 * the whole device, and cudaMalloc may). This call allocates nothing. Its
 * scratch (split partials and ticket counters) is a fixed device array
 * inside libqg of qg_decode_attention_static_scratch_capacity() bytes
 * (4 MiB) per device.
 *
 * Arguments, layouts and results as qg_decode_attention (same kernel, same
 * numerics); there is no ws / ws_bytes.
 * Limit: only shapes that merge through scratch (head_dim other than 32, 64,
 * 128 or 256, or more than 4 query heads per KV head) use the array; such a
 * shape whose scratch (qg_decode_attention_workspace_size) exceeds the fixed
 * capacity is refused with QG_ERR_WORKSPACE_TOO_SMALL before any launch (use
 * qg_decode_attention with a workspace for it). Cluster shapes use none and
 * are not limited.
 * Setup: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it; a failed
 * lookup returns QG_ERR_CUDA. Make the first call on a device before any
 * stream capture begins. A call that uses the array clears its ticket
 * counters (an async memset on `stream`) before the launch.
 * Concurrency: every call on one device shares the one scratch array, so
 * calls must not overlap in time: issue them on one stream, or order them
 * with events. Overlapping calls race on the scratch and give undefined
 * results. */
size_t qg_decode_attention_static_scratch_capacity(void);
qg_status qg_decode_attention_static_scratch(const float* q, const uint16_t* k_cache,
                                             const uint16_t* v_cache,
                                             const int32_t* kv_len, void* out,
                                             qg_dtype out_dtype, int B, int H,
                                             int Hkv, int D, int cap, float scale,
                                             void* stream);

/* ------------------------------------------------------------------------
 * Whole Qwen3 decode step  [TS: step; MK: Qwen3DecoderLayer::forward]
 * ---------------------------------------------------------------------- */
typedef struct qg_affine8_matrix {
  const uint32_t* w;       /* device uint32 [rows][cols/4] */
  const uint16_t* scales;  /* device bf16 [rows][cols/64] */
  const uint16_t* biases;  /* device bf16 [rows][cols/64] */
} qg_affine8_matrix;

typedef struct qg_qwen3_layer {
  const uint16_t* input_norm; /* device bf16 [hidden] */
  const uint16_t* post_norm;  /* device bf16 [hidden] */
  const uint16_t* q_norm;     /* device bf16 [head_dim] */
  const uint16_t* k_norm;     /* device bf16 [head_dim] */
  qg_affine8_matrix q;        /* [heads*head_dim][hidden] */
  qg_affine8_matrix k;        /* [kv_heads*head_dim][hidden] */
  qg_affine8_matrix v;        /* [kv_heads*head_dim][hidden] */
  qg_affine8_matrix o;        /* [hidden][heads*head_dim] */
  qg_affine8_matrix gate;     /* [ffn][hidden] */
  qg_affine8_matrix up;       /* [ffn][hidden] */
  qg_affine8_matrix down;     /* [hidden][ffn] */
} qg_qwen3_layer;

typedef struct qg_qwen3_config {
  int hidden, layers, heads, kv_heads, head_dim, ffn, vocab;
  float eps;     /* RMSNorm epsilon */
  double theta;  /* RoPE base */
} qg_qwen3_config;

typedef struct qg_qwen3_weights {
  qg_affine8_matrix embed;       /* tied embedding and LM head [vocab][hidden] */
  const uint16_t* final_norm;    /* device bf16 [hidden] */
  const qg_qwen3_layer* layers;  /* HOST array of cfg->layers entries */
} qg_qwen3_weights;

/* Workspace bytes for qg_decode_step at batch B and cache capacity cap. */
size_t qg_decode_step_workspace_size(const qg_qwen3_config* cfg, int B, int cap);

/* One decode step for B independent sequences sharing the weights.
 * For each sequence b: embed tokens[b]; run every layer at position
 * positions[b] (RMSNorm -> q,k,v -> per-head q/k RMSNorm -> RoPE -> K and V
 * written at cache row positions[b] -> attention over rows
 * [0, positions[b]] -> o_proj + residual -> RMSNorm -> gate, up -> SiLU-mul
 * -> down + residual); then the final RMSNorm and the tied LM head.
 * Execution: one launch per fused stage, chained with Programmatic Dependent
 * Launch (each GEMV streams its first weights while the previous kernel
 * finishes): the embedding, then per layer the q/k/v GEMV (input RMSNorm in
 * its prologue), attention (q/k norm, RoPE and the K/V append fused), o_proj
 * + residual, the gate/up GEMV (post-attention RMSNorm in its prologue), the
 * down GEMV (SiLU-mul in its prologue) + residual, then the LM head (final
 * RMSNorm in its prologue): 5 launches per layer plus 2. Nothing
 * synchronises or allocates, so a step can be captured in a CUDA graph.
 * Step graphs: on a stream other than the legacy or per-thread default
 * stream, and not while that stream is being captured, the call records
 * its launches into a CUDA graph the first time it sees this exact set of
 * arguments (every pointer and size, and the contents of *w and of its
 * layer table) and replays that graph on later calls with the same set: one
 * graph launch instead of ~140 kernel launches of host time. Up to 8 graphs
 * are kept, the least recently used dropped first; qg_step_graphs_enable(0)
 * turns this off and qg_step_graphs_clear() frees them. Results are the
 * same either way (the same kernels run).
 *
 * cfg, w      HOST structs (read during the call only).
 * k_cache, v_cache device bf16 [layers][B][kv_heads][cap][head_dim].
 * tokens, positions device int32 [B], read on the device. A sequence whose
 *             token is outside [0, vocab) or position outside [0, cap)
 *             gets NaN logits and its cache is not written.
 * logits      device fp32 [B][vocab].
 * ws          device workspace >= qg_decode_step_workspace_size(cfg,B,cap)
 *             bytes, 256-byte aligned; no initialisation needed (each step
 *             clears the attention counters with one small memset on
 *             `stream`).
 *             Use one workspace per stream at a time. On return its first
 *             B*hidden*4 bytes hold the residual stream after the last layer
 *             (fp32 [B][hidden], before the final norm).
 * Precision: residual stream, q/k/v and gate/up outputs and logits fp32;
 * norm outputs feeding a GEMV, cached K/V, attention output and SiLU-mul
 * output bf16.
 * Shape rules: hidden, heads*head_dim and ffn multiples of 64;
 * heads % kv_heads == 0, heads/kv_heads <= 8; head_dim % 32 == 0,
 * head_dim <= 256; 1 <= B <= 32; cap >= 1. */
qg_status qg_decode_step(const qg_qwen3_config* cfg, const qg_qwen3_weights* w,
                         uint16_t* k_cache, uint16_t* v_cache, int cap,
                         const int32_t* tokens, const int32_t* positions,
                         float* logits, int B, void* ws, size_t ws_bytes,
                         void* stream);

void qg_step_graphs_enable(int on);
void qg_step_graphs_clear(void);

/* Inspection aid (tests): byte offsets in the workspace of four bf16 arrays
 * that, after a step, hold the LAST decoder layer's values at its bf16
 * rounding points: offsets[0] the input-norm output [B][hidden], offsets[1]
 * the attention output [B][heads*head_dim], offsets[2] the
 * post-attention-norm output [B][hidden], offsets[3] the SiLU-mul output
 * [B][ffn]. */
qg_status qg_decode_step_inspect(const qg_qwen3_config* cfg, int B, int cap, size_t offsets[4]);

/* Inspection aid (tests): byte offsets in the workspace of six fp32 arrays
 * that, after a step, hold the LAST decoder layer's GEMV outputs:
 * offsets[0] q [B][heads*head_dim], offsets[1] k and offsets[2] v
 * [B][kv_heads*head_dim] (before the per-head norm and RoPE), offsets[3]
 * the residual stream after o_proj and its residual add [B][hidden],
 * offsets[4] gate and offsets[5] up [B][ffn]. */
qg_status qg_decode_step_inspect_f32(const qg_qwen3_config* cfg, int B, int cap,
                                     size_t offsets[6]);

/* ------------------------------------------------------------------------
 * Selected-token log-probability  [TS: compute_selected_logprob of the
 * greedy token; not printed on the page, read as the log-softmax]
 *   out[b] = logits[b][tokens[b]] - log(sum_i exp(logits[b][i])), in fp32
 *   with the row maximum subtracted first. A NaN logit or a token outside
 *   [0, V) gives NaN.
 * logits device fp32 [B][V]; tokens device int32 [B]; out device fp32 [B].
 * ws     >= qg_token_logprob_workspace_size(B, V) bytes, 8-byte aligned.
 * ---------------------------------------------------------------------- */
size_t qg_token_logprob_workspace_size(int B, int V);
qg_status qg_token_logprob(const float* logits, int B, int V, const int32_t* tokens,
                           float* out, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Token sampling  [MK: makima src/tts/qwen3, `sample_token` and
 * `apply_repetition_penalty`], in fp32 in the page's order:
 *   s = logits[b]; for each past[b][j] in [0, V), in order (every
 *   occurrence counts): s_t = s_t < 0 ? s_t * penalty : s_t / penalty;
 *   top_k == 0 or temperature == 0: out[b] = the first strict maximum of s
 *   (as qg_argmax_f32);
 *   otherwise: t = s / temperature; the k = min(top_k, V) largest t in
 *   descending order, equal values by index; e_j = exp(t_j - t_0);
 *   out[b] = the index of the first j whose running sum of e_j / sum(e)
 *   reaches r[b] (the first of the k if none does). NaN scores are never
 *   chosen.
 * logits  device fp32 [B][V] (not modified).
 * past    device int32 [B][P] or NULL with P = 0; entries outside [0, V)
 *         are skipped (use -1 for empty slots).
 * r       device fp32 [B], the uniform draws in [0, 1) (caller's random
 *         numbers); may be NULL for the greedy case.
 * out     device int32 [B].
 * Shape rules: 1 <= V; 0 <= top_k <= 64; ceil(V / 2048) * top_k <= 8192;
 * penalty > 0; temperature >= 0.
 * ws      >= qg_sample_workspace_size(B, V, top_k) bytes, 256-byte aligned.
 * ---------------------------------------------------------------------- */
size_t qg_sample_workspace_size(int B, int V, int top_k);
qg_status qg_sample(const float* logits, int B, int V, const int32_t* past, int P,
                    float penalty, float temperature, int top_k, const float* r,
                    int32_t* out, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Code predictor  [MK: makima src/tts/qwen3/code_predictor.rs,
 * CodePredictor::predict and CodePredictorLayer::forward]
 *
 * After the main model's LM head has chosen the group-0 code, the code
 * predictor chooses codes 1..groups-1 one after another. For each group g:
 *   x = input_proj @ bf16(concat(lm_hidden, embed_{g-1}(code[g-1])));
 *   the cfg->layers decoder layers on x, each with a fresh KV cache (so
 *   attention runs at position 0 over that one row);
 *   logits_g = heads[g] @ bf16(RMSNorm(x) * final_norm);
 *   code[g] = the first strict maximum of logits_g (as qg_argmax_f32).
 * Everything runs on the device with no host round trip between groups.
 *
 * cfg        HOST: hidden, layers, heads, kv_heads (= heads on the pages),
 *            head_dim, ffn, vocab = the codebook vocabulary, eps, theta;
 *            shape rules as qg_decode_step.
 * w          HOST struct: input_proj [hidden][2*hidden]; code_embed and
 *            heads point to HOST arrays of `groups` affine8 matrices
 *            [vocab][hidden] each (code_embed[g-1] embeds code g-1;
 *            heads[g] scores group g; code_embed[groups-1] and heads[0] are
 *            not used); layers a HOST array of cfg->layers layers;
 *            final_norm bf16 [hidden]; 2 <= groups <= 64.
 * lm_hidden  device fp32 [B][hidden]: the main model's last hidden state.
 * code0      device int32 [B]: the group-0 codes. A code outside [0, vocab)
 *            gives NaN logits downstream.
 * codes      device int32 [groups][B] out; codes[0] = code0.
 * logits     device fp32 [groups][B][vocab] out, or NULL: logits of group
 *            g >= 1 in row g (row 0 not written).
 * ws         >= qg_code_predict_workspace_size(cfg, B) bytes, 256-byte
 *            aligned; no initialisation needed.
 * Like qg_decode_step, on a non-default stream the call is recorded into a
 * CUDA graph once and replayed (qg_step_graphs_enable / _clear apply). */
typedef struct qg_code_predictor_weights {
  qg_affine8_matrix input_proj;
  const qg_affine8_matrix* code_embed;
  const qg_affine8_matrix* heads;
  const qg_qwen3_layer* layers;
  const uint16_t* final_norm;
  int groups;
} qg_code_predictor_weights;

size_t qg_code_predict_workspace_size(const qg_qwen3_config* cfg, int B);
qg_status qg_code_predict(const qg_qwen3_config* cfg, const qg_code_predictor_weights* w,
                          const float* lm_hidden, const int32_t* code0, int32_t* codes,
                          float* logits, int B, void* ws, size_t ws_bytes, void* stream);

/* Inspection aid (tests): qg_code_predict that also writes a trace of every
 * group's layers to `trace` (device, 256-byte aligned, at least out[0] bytes
 * of qg_code_predict_trace_layout). Layout, with out[] from that call:
 * group g (1 .. groups-1) starts at (g-1) * out[1] and holds the bf16
 * concatenated input [B][2 hidden] at offset 0, then slots s = 0 ..
 * cfg->layers at out[2] + s * out[3]. Slot 0 is taken after input_proj,
 * slot s >= 1 after layer s-1. A slot is a copy of the workspace head: the
 * residual stream fp32 [B][hidden] at offset 0 and the other step buffers
 * at the offsets qg_decode_step_inspect and qg_decode_step_inspect_f32
 * give for (cfg, B, cap = 1), so that slot s >= 1 holds layer s-1's values;
 * then the K row and the V row that layer wrote (bf16 [B][kv_heads]
 * [head_dim] each, the second starting where the first is rounded up to 256
 * bytes). The copies are ordinary stream copies between the launches: the
 * results are those of qg_code_predict. */
qg_status qg_code_predict_trace_layout(const qg_qwen3_config* cfg, int B, int groups,
                                       size_t out[4]);
qg_status qg_code_predict_traced(const qg_qwen3_config* cfg, const qg_code_predictor_weights* w,
                                 const float* lm_hidden, const int32_t* code0, int32_t* codes,
                                 float* logits, int B, void* ws, size_t ws_bytes, void* trace,
                                 size_t trace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Greedy token  [TS: turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs, `argmax`]
 *   out[b] = index of the first strict maximum of logits[b][0..V), NaNs
 *   skipped; 0 when no value beats -inf (all -inf or NaN). -0 and +0 are
 *   equal (the first wins). The result is exact and deterministic.
 *
 * logits  device fp32 [B][V], 4-byte aligned.
 * out     device int32 [B].
 * ws      device workspace >= qg_argmax_workspace_size(B, V) bytes, 8-byte
 *         aligned; no initialisation needed.
 * Two launches on `stream`; 1 <= V, 0 <= B (B = 0 does nothing).
 * ---------------------------------------------------------------------- */
size_t qg_argmax_workspace_size(int B, int V);
qg_status qg_argmax_f32(const float* logits, int B, int V, int32_t* out, void* ws,
                        size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Affine-INT8 group-64 matmul on the tcgen05 tensor cores: the linears of
 * many activation rows at once (a batched prefill, a batched decode step)
 * [TS: PackedLinear / load_packed_linear; the prompt rows of
 * transcribe_with_details]
 *
 *   y[t][r] = sum_c (q[r][c] * s[r][c/64] + beta[r][c/64]) * x[t][c]
 *             (+ residual[t][r])
 *
 * w, scales, biases as qg_gemv_affine8_g64 ([N][K]); x device bf16 [T][K]
 * (16-byte aligned); y device [T][N] of y_dtype (may alias residual);
 * residual device fp32 [T][N] or NULL (only with a fp32 y).
 * The weights are dequantized in fp32 and split into two bf16 halves
 * (hi + lo carries w to about 2^-18 relative); both are multiplied with the
 * bf16 x, fp32 accumulation in tensor memory.
 * ws       device, >= 4 bytes, 4-byte aligned: the error word (cleared by
 *          the call; nonzero after a device-side wait gave up (1 s bound);
 *          read it with qg_gemm_q4_0_error(0, 0, ws, ...)).
 * Shape rules: K % 64 == 0, T >= 0, N >= 0.
 * ---------------------------------------------------------------------- */
qg_status qg_gemm_affine8_g64(const uint32_t* w, const uint16_t* scales, const uint16_t* biases,
                              const uint16_t* x, void* y, qg_dtype y_dtype,
                              const float* residual, int N, int K, int T, void* ws,
                              size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Batched prefill of one sequence  [TS: transcribe_with_details, the prompt
 * rows through `step`; MK: Qwen3Model::forward with causal_mask]
 *
 * The T prompt rows tokens[0..T) at positions p0 .. p0+T-1 go through every
 * layer together, in qg_decode_step's op order and precision points, with
 * the linears on qg_gemm_affine8_g64's tensor-core matmul: embedding rows;
 * per layer RMSNorm, q/k/v (one launch), per-head q/k RMSNorm + NeoX RoPE
 * with K and V rows written to the cache at p0 + t, causal attention of
 * every row over the cached rows [0, p0) and the prompt rows up to itself
 * (qg_attention_rows' kernel reading the cache), o_proj + residual,
 * RMSNorm, gate/up (one launch), SiLU-mul, down + residual; then the final
 * RMSNorm and the tied LM head for the last row.
 * cfg, w      HOST structs as qg_decode_step (head_dim 64 or 128).
 * k_cache, v_cache device bf16 [layers][1][kv_heads][cap][head_dim]: rows
 *             [0, p0) must hold the earlier rows; rows p0 .. p0+T-1 are
 *             written (not for a token outside [0, vocab), whose row is NaN).
 * tokens      device int32 [T].  Requires 0 <= p0, p0 + T <= cap.
 * logits      device fp32 [vocab] (the last row's), or NULL.
 * ws          >= qg_prefill_workspace_size(cfg, T) bytes, 256-byte aligned.
 *             qg_prefill_inspect gives the byte offsets of the LAST layer's
 *             values after a call: [0] the residual stream fp32 [T][hidden]
 *             (after that layer), [1] input-norm output bf16 [T][hidden],
 *             [2] q fp32 [T][heads*head_dim], [3] k and [4] v fp32
 *             [T][kv_heads*head_dim], [5] normed and roped q bf16
 *             [T][heads*head_dim], [6] attention output bf16, [7] residual
 *             after o_proj fp32 [T][hidden], [8] post-norm output bf16,
 *             [9] gate and [10] up fp32 [T][ffn], [11] SiLU-mul output bf16.
 * ---------------------------------------------------------------------- */
size_t qg_prefill_workspace_size(const qg_qwen3_config* cfg, int T);
qg_status qg_prefill(const qg_qwen3_config* cfg, const qg_qwen3_weights* w, uint16_t* k_cache,
                     uint16_t* v_cache, int cap, const int32_t* tokens, int T, int p0,
                     float* logits, void* ws, size_t ws_bytes, void* stream);
qg_status qg_prefill_inspect(const qg_qwen3_config* cfg, int T, size_t offsets[12]);

/* ------------------------------------------------------------------------
 * LayerNorm  [FT: layer_norm_affine (layer_norm_last_dim, then * g + b)]
 *   y[r][i] = (x[r][i] - mean_r) / sqrt(var_r + eps) * gamma[i] + beta[i],
 *   mean and biased variance over the row, in fp32.
 * x device fp32 [rows][dim]; gamma, beta device fp32 [dim]; y device
 * [rows][dim] of y_dtype (rounded to nearest even for QG_BF16). All 16-byte
 * aligned. Shape rules: dim % 4 == 0, 4 <= dim <= 2048.
 * ---------------------------------------------------------------------- */
qg_status qg_layernorm(const float* x, const float* gamma, const float* beta, float eps,
                       void* y, qg_dtype y_dtype, int rows, int dim, void* stream);

/* ------------------------------------------------------------------------
 * Softmax attention of many query rows  [FT: multi_head_attn; MK:
 * Qwen3Attention::forward with causal_mask and repeat_kv]
 *   out[b][t][h] = sum_s softmax_s(q[b][t][h] . k[b][s][kv] / sqrt(D)) v[b][s][kv],
 *   kv = h / (H / Hkv); s over all S keys, or with `causal` over
 *   s <= S - T + t (row t at position S - T + t, after S - T earlier keys).
 * q, out   device bf16 [B][T][H][D];  k, v device bf16 [B][S][Hkv][D].
 * Tensor cores (bf16 operands, fp32 accumulation); the softmax weights are
 * rounded to bf16 for the weighted sum of V (and summed as rounded), out is
 * rounded to bf16. All pointers 16-byte aligned.
 * Shape rules: D = 64 or 128, H % Hkv == 0, causal needs T <= S; S = 0
 * gives zero rows (k and v are then not read and may be NULL).
 * ---------------------------------------------------------------------- */
qg_status qg_attention_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                            uint16_t* out, int B, int T, int S, int H, int Hkv, int D,
                            int causal, void* stream);

/* ------------------------------------------------------------------------
 * Whisper encoder layer  [FT: encoder_layer, pre-LayerNorm]
 *   a = LN1(x); q = a Wq^T + bq; k = a Wk^T; v = a Wv^T + bv;
 *   x1 = x + attention(q, k, v) Wo^T + bo        (every frame to every frame)
 *   x  = x1 + gelu_tanh(LN2(x1) W1^T + b1) W2^T + b2
 * The six matrices are Q4_0 blocks (qg_gemm_q4_0 layout) multiplied on the
 * tensor cores with bf16 operands; the LN outputs, q, k, v, the attention
 * output and the GELU output are stored as bf16; the residual stream is
 * fp32. Nine launches: qg_layernorm, three qg_gemm_q4_0_ex (bf16 out),
 * qg_attention_rows, qg_gemm_q4_0_ex with the residual (into x1),
 * qg_layernorm, fc1 with GELU (bf16 out), fc2 with the residual (into x).
 * cfg, w     HOST structs. LN vectors and biases device fp32 (LN vectors
 *            16-byte aligned); matrices device Q4_0 [out][(in/32)*18].
 * x          device fp32 [M][d_model], 16-byte aligned: input, then output.
 * ws         >= qg_whisper_encoder_layer_workspace_size(cfg, M) bytes,
 *            256-byte aligned; qg_whisper_encoder_layer_inspect gives the
 *            byte offsets of a (bf16 [M][d]), q, k, v, the attention output
 *            (bf16), x1 (fp32 [M][d]), LN2's output (bf16), the GELU output
 *            (bf16 [M][ffn]) and, 9th, the six matmuls' error words (256
 *            bytes apart; read with qg_gemm_q4_0_error(0, 0, ws + off + 256 i)).
 * Shape rules: d_model and ffn multiples of 128, d_model <= 2048, head size
 * d_model / heads of 64 or 128.
 * ---------------------------------------------------------------------- */
typedef struct qg_whisper_config {
  int d_model, heads, ffn;
  float eps;  /* LayerNorm epsilon (1e-5 on the page) */
} qg_whisper_config;

typedef struct qg_whisper_layer {
  const float* ln1_g;
  const float* ln1_b;
  const uint8_t* q;
  const float* q_b;
  const uint8_t* k;   /* k_proj has no bias */
  const uint8_t* v;
  const float* v_b;
  const uint8_t* o;
  const float* o_b;
  const float* ln2_g;
  const float* ln2_b;
  const uint8_t* fc1;
  const float* fc1_b;
  const uint8_t* fc2;
  const float* fc2_b;
} qg_whisper_layer;

size_t qg_whisper_encoder_layer_workspace_size(const qg_whisper_config* cfg, int M);
qg_status qg_whisper_encoder_layer(const qg_whisper_config* cfg, const qg_whisper_layer* w,
                                   float* x, int M, void* ws, size_t ws_bytes, void* stream);
qg_status qg_whisper_encoder_layer_inspect(const qg_whisper_config* cfg, int M,
                                           size_t offsets[9]);

/* ------------------------------------------------------------------------
 * Timeline (diagnostics). The pages have no counterpart. In a library built
 * with QG_TIMELINE (libqg_timeline.so; the default build records nothing
 * and qg_timeline_available() returns 0), the decode step's kernels launched
 * between qg_timeline_begin and qg_timeline_end each fill one record of
 * `records` (device, 16-byte aligned, cap records of 32 bytes, zero-filled
 * by the caller) when they run, also from a CUDA graph captured meanwhile:
 * four uint64 per launch -- the bitwise complement of the earliest CTA
 * entry, the latest return from the wait for the previous kernel, the
 * latest CTA exit (all %globaltimer nanoseconds, maxima over the launch's
 * CTAs), and the latest CTA entry. qg_timeline_end stops recording, copies the
 * launch kinds (1 embedding, 2 q/k/v GEMV, 3 attention, 4 o_proj, 5 gate/up,
 * 6 down, 7 output head, 8 other) of the first max_kinds launches to kinds
 * (host, may be NULL) and returns the number of launches recorded.
 * ---------------------------------------------------------------------- */
int qg_timeline_available(void);
qg_status qg_timeline_begin(void* records, int cap);
int qg_timeline_end(int* kinds, int max_kinds);

/* ------------------------------------------------------------------------
 * Test exports: the unpack and dequant the kernels use, written out.
 * ---------------------------------------------------------------------- */
/* q[r][c] as fp32 (0..255) from packed words; out device fp32 [N][K]. */
qg_status qg_unpack_affine8(const uint32_t* w, float* out, int N, int K, void* stream);
/* q*s+beta as fp32 (one rounding); out device fp32 [N][K]. */
qg_status qg_dequant_affine8_g64(const uint32_t* w, const uint16_t* scales,
                                 const uint16_t* biases, float* out, int N,
                                 int K, void* stream);
/* d*(n-8) as fp32 (exact); out device fp32 [N][K]. */
qg_status qg_dequant_q4_0(const uint8_t* blocks, float* out, int N, int K,
                          void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QG_H */
