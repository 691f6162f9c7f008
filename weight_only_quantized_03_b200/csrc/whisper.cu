// The Whisper encoder layer around the Q4_0 tensor-core matmul.
//
// Definition: fuel-transformers 0.19.1, src/models/lazy_quantized_whisper.rs,
// `encoder_layer` (pre-LayerNorm):
//   x_ln = LayerNorm(x; ln1, eps 1e-5)
//   q = x_ln Wq^T + bq,  k = x_ln Wk^T (no bias),  v = x_ln Wv^T + bv
//   ctx = softmax(q k^T / sqrt(d_head)) v per head, every frame to every frame
//   x = x + (ctx Wo^T + bo)
//   x_ln = LayerNorm(x; ln2, eps 1e-5)
//   x = x + (gelu_tanh(x_ln W1^T + b1) W2^T + b2)
// (`layer_norm_affine`, `q_linear`, `multi_head_attn`.) The matmuls run on
// the tcgen05 GEMM with bf16 operands; the LayerNorm outputs, q/k/v, the
// attention output and the GELU output are stored as bf16 (the operands of
// the next tensor-core product); the residual stream stays fp32.
//
// Launches: LayerNorm, the q, k and v matmuls (bf16 out, bias in the
// epilogue), attention (attention_rows.cu), the out projection with bias and
// the residual add in its epilogue, LayerNorm, fc1 with bias and GELU in its
// epilogue (bf16 out), fc2 with bias and the residual add (into x).
#include "qg_internal.cuh"

namespace qg {

// LayerNorm of one row per warp: the row is held in registers (VPL float4 a
// lane), mean and biased variance in two passes over the registers (warp
// sums, fixed order), y = (x - mean) / sqrt(var + eps) * gamma + beta.
template <int VPL>
__global__ void __launch_bounds__(256) layernorm_kernel(const float* __restrict__ x,
                                                        const float* __restrict__ gamma,
                                                        const float* __restrict__ beta, float eps,
                                                        void* __restrict__ y, int y_bf16, int rows,
                                                        int dim) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)warp * dim);
  const int n4 = dim / 4;
  float4 v[VPL];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int j = lane + 32 * i;
    v[i] = j < n4 ? __ldg(xr + j) : make_float4(0.f, 0.f, 0.f, 0.f);
    s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
  }
  const float mean = warp_sum(s) / (float)dim;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    if (lane + 32 * i < n4) {
      const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
      q += (a * a + b * b) + (c * c + d * d);
    }
  }
  const float inv = 1.0f / sqrtf(warp_sum(q) / (float)dim + eps);
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int j = lane + 32 * i;
    if (j >= n4) break;
    const float4 g = __ldg(reinterpret_cast<const float4*>(gamma) + j);
    const float4 bb = __ldg(reinterpret_cast<const float4*>(beta) + j);
    const float o0 = (v[i].x - mean) * inv * g.x + bb.x, o1 = (v[i].y - mean) * inv * g.y + bb.y;
    const float o2 = (v[i].z - mean) * inv * g.z + bb.z, o3 = (v[i].w - mean) * inv * g.w + bb.w;
    const size_t o = (size_t)warp * dim + 4 * j;
    if (y_bf16)
      *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(y) + o) =
          make_uint2((uint32_t)f32_to_bf16_bits(o0) | ((uint32_t)f32_to_bf16_bits(o1) << 16),
                     (uint32_t)f32_to_bf16_bits(o2) | ((uint32_t)f32_to_bf16_bits(o3) << 16));
    else
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + o) = make_float4(o0, o1, o2, o3);
  }
}

cudaError_t layernorm_launch(const float* x, const float* g, const float* b, float eps, void* y,
                             bool y_bf16, int rows, int dim, cudaStream_t st) {
  const dim3 grid((rows + 7) / 8), block(256);
  const int vpl = (dim / 4 + 31) / 32;
  if (vpl <= 4)
    return launch_pdl(layernorm_kernel<4>, grid, block, 0, st, false, x, g, b, eps, y,
                      (int)y_bf16, rows, dim);
  if (vpl <= 8)
    return launch_pdl(layernorm_kernel<8>, grid, block, 0, st, false, x, g, b, eps, y,
                      (int)y_bf16, rows, dim);
  return launch_pdl(layernorm_kernel<16>, grid, block, 0, st, false, x, g, b, eps, y,
                    (int)y_bf16, rows, dim);
}

}  // namespace qg

using namespace qg;

extern "C" qg_status qg_layernorm(const float* x, const float* gamma, const float* beta, float eps,
                                  void* y, qg_dtype y_dtype, int rows, int dim, void* stream) {
  clear_error();
  QG_REQUIRE(rows >= 0 && dim >= 4 && dim % 4 == 0 && dim <= 2048, QG_ERR_UNSUPPORTED_SHAPE,
             "qg_layernorm: rows=%d dim=%d (dim a multiple of 4 in [4, 2048])", rows, dim);
  QG_REQUIRE(y_dtype == QG_F32 || y_dtype == QG_BF16, QG_ERR_INVALID_ARGUMENT,
             "qg_layernorm: y_dtype=%d", (int)y_dtype);
  QG_REQUIRE(eps >= 0.f, QG_ERR_INVALID_ARGUMENT, "qg_layernorm: eps must be >= 0");
  if (rows == 0) return QG_OK;
  QG_REQUIRE(x && gamma && beta && y, QG_ERR_INVALID_ARGUMENT, "qg_layernorm: null pointer");
  QG_REQUIRE(aligned(x, 16) && aligned(gamma, 16) && aligned(beta, 16) && aligned(y, 16),
             QG_ERR_MISALIGNED, "qg_layernorm: x, gamma, beta and y must be 16-byte aligned");
  layernorm_launch(x, gamma, beta, eps, y, y_dtype == QG_BF16, rows, dim, (cudaStream_t)stream);
  return check_launch("qg_layernorm");
}

// --------------------------------------------------------------------------
// The whole layer.
// --------------------------------------------------------------------------

namespace {

struct WLayout {
  size_t xl, q, k, v, ctx, xa, xl2, mid, err, total;
};

WLayout wlayout(const qg_whisper_config& c, int M) {
  WLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  const size_t md = (size_t)M * c.d_model;
  L.xl = take(md * 2);
  L.q = take(md * 2);
  L.k = take(md * 2);
  L.v = take(md * 2);
  L.ctx = take(md * 2);
  L.xa = take(md * 4);
  L.xl2 = take(md * 2);
  L.mid = take((size_t)M * c.ffn * 2);
  L.err = take(6 * 256);  // one error word per matmul, 256 bytes apart
  L.total = off;
  return L;
}

qg_status check_cfg(const qg_whisper_config* c, int M, const char* what) {
  QG_REQUIRE(c, QG_ERR_INVALID_ARGUMENT, "%s: cfg is NULL", what);
  QG_REQUIRE(M >= 0, QG_ERR_UNSUPPORTED_SHAPE, "%s: M=%d", what, M);
  QG_REQUIRE(c->heads >= 1 && c->d_model % c->heads == 0 &&
                 (c->d_model / c->heads == 64 || c->d_model / c->heads == 128),
             QG_ERR_UNSUPPORTED_SHAPE, "%s: d_model=%d heads=%d (head size 64 or 128)", what,
             c->d_model, c->heads);
  QG_REQUIRE(c->d_model % 128 == 0 && c->d_model <= 2048 && c->ffn % 128 == 0 && c->ffn > 0,
             QG_ERR_UNSUPPORTED_SHAPE,
             "%s: d_model=%d (a multiple of 128, <= 2048) and ffn=%d (a multiple of 128)", what,
             c->d_model, c->ffn);
  QG_REQUIRE(c->eps >= 0.f, QG_ERR_INVALID_ARGUMENT, "%s: eps < 0", what);
  return QG_OK;
}

}  // namespace

extern "C" size_t qg_whisper_encoder_layer_workspace_size(const qg_whisper_config* cfg, int M) {
  if (!cfg || M < 0) return 0;
  return wlayout(*cfg, M).total;
}

extern "C" qg_status qg_whisper_encoder_layer_inspect(const qg_whisper_config* cfg, int M,
                                                     size_t offsets[9]) {
  clear_error();
  qg_status st = check_cfg(cfg, M, "qg_whisper_encoder_layer_inspect");
  if (st != QG_OK) return st;
  QG_REQUIRE(offsets, QG_ERR_INVALID_ARGUMENT, "qg_whisper_encoder_layer_inspect: null offsets");
  const WLayout L = wlayout(*cfg, M);
  const size_t o[9] = {L.xl, L.q, L.k, L.v, L.ctx, L.xa, L.xl2, L.mid, L.err};
  for (int i = 0; i < 9; ++i) offsets[i] = o[i];
  return QG_OK;
}

extern "C" qg_status qg_whisper_encoder_layer(const qg_whisper_config* cfg,
                                              const qg_whisper_layer* w, float* x, int M, void* ws,
                                              size_t ws_bytes, void* stream) {
  const char* what = "qg_whisper_encoder_layer";
  clear_error();
  qg_status st = check_cfg(cfg, M, what);
  if (st != QG_OK) return st;
  const qg_whisper_config& c = *cfg;
  QG_REQUIRE(w, QG_ERR_INVALID_ARGUMENT, "%s: weights is NULL", what);
  QG_REQUIRE(w->ln1_g && w->ln1_b && w->q && w->q_b && w->k && w->v && w->v_b && w->o && w->o_b &&
                 w->ln2_g && w->ln2_b && w->fc1 && w->fc1_b && w->fc2 && w->fc2_b,
             QG_ERR_INVALID_ARGUMENT, "%s: a weight pointer is NULL", what);
  for (const void* p : {(const void*)w->ln1_g, (const void*)w->ln1_b, (const void*)w->ln2_g,
                        (const void*)w->ln2_b})
    QG_REQUIRE(aligned(p, 16), QG_ERR_MISALIGNED, "%s: LayerNorm vectors must be 16-byte aligned",
               what);
  for (const void* p : {(const void*)w->q, (const void*)w->k, (const void*)w->v, (const void*)w->o,
                        (const void*)w->fc1, (const void*)w->fc2})
    QG_REQUIRE(aligned(p, 2), QG_ERR_MISALIGNED, "%s: Q4_0 blocks must be 2-byte aligned", what);
  for (const void* p : {(const void*)w->q_b, (const void*)w->v_b, (const void*)w->o_b,
                        (const void*)w->fc1_b, (const void*)w->fc2_b})
    QG_REQUIRE(aligned(p, 4), QG_ERR_MISALIGNED, "%s: biases must be 4-byte aligned", what);
  if (M == 0) return QG_OK;
  QG_REQUIRE(x && aligned(x, 16), QG_ERR_INVALID_ARGUMENT, "%s: x NULL or not 16-byte aligned",
             what);
  const WLayout L = wlayout(c, M);
  QG_REQUIRE(ws && ws_bytes >= L.total, QG_ERR_WORKSPACE_TOO_SMALL,
             "%s: workspace of %zu bytes given, %zu needed", what, ws_bytes, L.total);
  QG_REQUIRE(aligned(ws, 256), QG_ERR_MISALIGNED, "%s: ws not 256-byte aligned", what);

  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  uint16_t* xl = reinterpret_cast<uint16_t*>(base + L.xl);
  uint16_t* q = reinterpret_cast<uint16_t*>(base + L.q);
  uint16_t* k = reinterpret_cast<uint16_t*>(base + L.k);
  uint16_t* v = reinterpret_cast<uint16_t*>(base + L.v);
  uint16_t* ctx = reinterpret_cast<uint16_t*>(base + L.ctx);
  float* xa = reinterpret_cast<float*>(base + L.xa);
  uint16_t* xl2 = reinterpret_cast<uint16_t*>(base + L.xl2);
  uint16_t* mid = reinterpret_cast<uint16_t*>(base + L.mid);
  uint8_t* err = base + L.err;
  int gi = 0;  // which matmul: its error word
  const int d = c.d_model, F = c.ffn;
  auto gemm = [&](const uint8_t* W, const void* A, const float* bias, const float* res, void* C,
                  qg_dtype cdt, int gelu, int N, int K) {
    return qg_gemm_q4_0_ex(W, A, QG_BF16, bias, res, C, cdt, gelu, M, N, K, err + 256 * gi++, 256,
                           stream);
  };
  layernorm_launch(x, w->ln1_g, w->ln1_b, c.eps, xl, true, M, d, s);
  if ((st = gemm(w->q, xl, w->q_b, nullptr, q, QG_BF16, 0, d, d)) != QG_OK) return st;
  if ((st = gemm(w->k, xl, nullptr, nullptr, k, QG_BF16, 0, d, d)) != QG_OK) return st;
  if ((st = gemm(w->v, xl, w->v_b, nullptr, v, QG_BF16, 0, d, d)) != QG_OK) return st;
  qg_status a = qg_attention_rows(q, k, v, ctx, 1, M, M, c.heads, c.heads, d / c.heads, 0, stream);
  if (a != QG_OK) return a;
  if ((st = gemm(w->o, ctx, w->o_b, x, xa, QG_F32, 0, d, d)) != QG_OK) return st;
  layernorm_launch(xa, w->ln2_g, w->ln2_b, c.eps, xl2, true, M, d, s);
  if ((st = gemm(w->fc1, xl2, w->fc1_b, nullptr, mid, QG_BF16, 1, F, d)) != QG_OK) return st;
  if ((st = gemm(w->fc2, mid, w->fc2_b, xa, x, QG_F32, 0, d, F)) != QG_OK) return st;
  return check_launch(what);
}
