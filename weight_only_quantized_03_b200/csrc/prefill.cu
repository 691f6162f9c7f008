// Batched prefill: the prompt rows of one sequence through every layer at
// once, on the tensor-core matmul (gemm_affine8_sm100.cu).
//
// Definition: turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs,
// `transcribe_with_details` runs the prompt rows one after another through
// `step`; makima src/tts/qwen3/model.rs, `Qwen3Model::forward` with
// `causal_mask`, runs them together: row t (at position p0 + t) attends to the
// cached rows [0, p0) and to the prompt rows up to itself. Both give the same
// values (the incremental cache equals the full-prefix recompute), so the
// rows are taken together here, in the decode step's op order and precision
// points:
//   x = embed(tokens)                                   fp32 [T][hidden]
//   per layer: xn = bf16(RMSNorm(x)); q, k, v = W xn (fp32);
//     per-head q/k RMSNorm, NeoX RoPE at p0 + t; K, V rows bf16 into the
//     cache at p0 + t; attention (causal, GQA) -> bf16; xa = x + W_o att;
//     xn2 = bf16(RMSNorm(xa)); gate, up = W xn2; h = bf16(silu(gate) up);
//     x = xa + W_down h
//   then the final RMSNorm and the tied LM head for the last row.
// A row whose token is outside [0, vocab) gets NaN values and writes nothing
// to the cache.
#include "attention_body.cuh"
#include "attention_rows.cuh"

namespace qg {

// Row t of the prompt: query heads normed and roped into qb (bf16), key
// heads normed and roped and value heads rounded into the cache at row
// p0 + t. One warp per head; grid (T, ceil((H + 2 Hkv) / 8)).
__global__ void __launch_bounds__(256)
    prefill_qk_kernel(const float* __restrict__ q, const float* __restrict__ k,
                      const float* __restrict__ v, const uint16_t* __restrict__ qn,
                      const uint16_t* __restrict__ kn, const int32_t* __restrict__ tok, int vocab,
                      float eps, double theta, int p0, uint16_t* __restrict__ qb,
                      uint16_t* __restrict__ kc, uint16_t* __restrict__ vc, int H, int Hkv, int D,
                      int cap) {
  __shared__ float2 cs[128];
  const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pos = p0 + t;
  for (int i = threadIdx.x; i < D / 2; i += blockDim.x) {
    const double inv_freq = pow(theta, -2.0 * (double)i / (double)D);
    double sd, cd;
    sincos((double)pos * inv_freq, &sd, &cd);
    cs[i] = make_float2((float)cd, (float)sd);
  }
  __syncthreads();
  const int j = blockIdx.y * 8 + warp;
  const int tk = tok[t];
  const bool write = tk >= 0 && tk < vocab;
  if (j < H) {
    uint16_t* dst = qb + ((size_t)t * H + j) * D;
    norm_rope_head<true>(q + ((size_t)t * H + j) * D, qn, D, eps, cs, lane,
                   [&](int i, float r) { dst[i] = f32_to_bf16_bits(r); });
  } else if (j < H + Hkv) {
    const int h = j - H;
    uint16_t* dst = kc + ((size_t)h * cap + pos) * D;
    norm_rope_head<true>(k + ((size_t)t * Hkv + h) * D, kn, D, eps, cs, lane, [&](int i, float r) {
      if (write) dst[i] = f32_to_bf16_bits(r);
    });
  } else if (j < H + 2 * Hkv) {
    const int h = j - H - Hkv;
    uint16_t* dst = vc + ((size_t)h * cap + pos) * D;
    const float* src = v + ((size_t)t * Hkv + h) * D;
    for (int d = lane; d < D; d += 32)
      if (write) dst[d] = f32_to_bf16_bits(src[d]);
  }
}

struct PrefillLayout {
  size_t x, xn, q, k, v, qb, att, xa, xn2, gate, up, h, err, total;
};

static size_t pa256(size_t v) { return (v + 255) & ~(size_t)255; }

static PrefillLayout prefill_layout(const qg_qwen3_config& c, int T) {
  PrefillLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += pa256(bytes);
    return o;
  };
  const size_t HD = (size_t)c.heads * c.head_dim, KD = (size_t)c.kv_heads * c.head_dim;
  L.x = take((size_t)T * c.hidden * 4);
  L.xn = take((size_t)T * c.hidden * 2);
  L.q = take((size_t)T * HD * 4);
  L.k = take((size_t)T * KD * 4);
  L.v = take((size_t)T * KD * 4);
  L.qb = take((size_t)T * HD * 2);
  L.att = take((size_t)T * HD * 2);
  L.xa = take((size_t)T * c.hidden * 4);
  L.xn2 = take((size_t)T * c.hidden * 2);
  L.gate = take((size_t)T * c.ffn * 4);
  L.up = take((size_t)T * c.ffn * 4);
  L.h = take((size_t)T * c.ffn * 2);
  L.err = take(256);
  L.total = off;
  return L;
}

}  // namespace qg

using namespace qg;

static qg_status prefill_check(const qg_qwen3_config* c, int T, const char* what) {
  QG_REQUIRE(c, QG_ERR_INVALID_ARGUMENT, "%s: cfg is NULL", what);
  QG_REQUIRE(T >= 0, QG_ERR_UNSUPPORTED_SHAPE, "%s: T=%d", what, T);
  QG_REQUIRE(c->hidden > 0 && c->hidden % 64 == 0 && c->ffn > 0 && c->ffn % 64 == 0 &&
                 c->layers >= 0 && c->vocab >= 1,
             QG_ERR_UNSUPPORTED_SHAPE, "%s: hidden=%d ffn=%d layers=%d vocab=%d", what, c->hidden,
             c->ffn, c->layers, c->vocab);
  QG_REQUIRE(c->heads >= 1 && c->kv_heads >= 1 && c->heads % c->kv_heads == 0,
             QG_ERR_UNSUPPORTED_SHAPE, "%s: heads=%d kv_heads=%d", what, c->heads, c->kv_heads);
  QG_REQUIRE(c->head_dim == 64 || c->head_dim == 128, QG_ERR_UNSUPPORTED_SHAPE,
             "%s: head_dim=%d must be 64 or 128", what, c->head_dim);
  QG_REQUIRE(((long long)c->heads * c->head_dim) % 64 == 0, QG_ERR_UNSUPPORTED_SHAPE,
             "%s: heads*head_dim must be a multiple of 64", what);
  QG_REQUIRE(c->eps >= 0.f && c->theta > 0.0, QG_ERR_INVALID_ARGUMENT, "%s: eps/theta", what);
  return QG_OK;
}

extern "C" size_t qg_prefill_workspace_size(const qg_qwen3_config* cfg, int T) {
  if (!cfg || T < 0 || cfg->heads < 1 || cfg->kv_heads < 1) return 0;
  return prefill_layout(*cfg, T).total;
}

extern "C" qg_status qg_prefill_inspect(const qg_qwen3_config* cfg, int T, size_t offsets[12]) {
  clear_error();
  qg_status st = prefill_check(cfg, T, "qg_prefill_inspect");
  if (st != QG_OK) return st;
  QG_REQUIRE(offsets, QG_ERR_INVALID_ARGUMENT, "qg_prefill_inspect: null offsets");
  const PrefillLayout L = prefill_layout(*cfg, T);
  const size_t o[12] = {L.x, L.xn, L.q, L.k, L.v, L.qb, L.att, L.xa, L.xn2, L.gate, L.up, L.h};
  for (int i = 0; i < 12; ++i) offsets[i] = o[i];
  return QG_OK;
}

extern "C" qg_status qg_prefill(const qg_qwen3_config* cfg, const qg_qwen3_weights* w,
                                uint16_t* k_cache, uint16_t* v_cache, int cap,
                                const int32_t* tokens, int T, int p0, float* logits, void* ws,
                                size_t ws_bytes, void* stream) {
  const char* what = "qg_prefill";
  clear_error();
  qg_status st = prefill_check(cfg, T, what);
  if (st != QG_OK) return st;
  const qg_qwen3_config& c = *cfg;
  QG_REQUIRE(p0 >= 0 && cap >= 1 && (long long)p0 + T <= cap, QG_ERR_UNSUPPORTED_SHAPE,
             "%s: rows [p0=%d, p0+T=%d) must lie in the cache (cap=%d)", what, p0, p0 + T, cap);
  if (T == 0) return QG_OK;
  QG_REQUIRE(w && (c.layers == 0 || w->layers) && w->embed.w && w->embed.scales &&
                 w->embed.biases && w->final_norm,
             QG_ERR_INVALID_ARGUMENT, "%s: null weights", what);
  for (int l = 0; l < c.layers; ++l) {
    const qg_qwen3_layer& L = w->layers[l];
    for (const qg_affine8_matrix* m : {&L.q, &L.k, &L.v, &L.o, &L.gate, &L.up, &L.down}) {
      QG_REQUIRE(m->w && m->scales && m->biases, QG_ERR_INVALID_ARGUMENT,
                 "%s: layer %d has a null matrix", what, l);
      QG_REQUIRE(aligned(m->w, 16) && aligned(m->scales, 2) && aligned(m->biases, 2),
                 QG_ERR_MISALIGNED, "%s: layer %d matrix misaligned", what, l);
    }
    QG_REQUIRE(L.input_norm && L.post_norm && L.q_norm && L.k_norm, QG_ERR_INVALID_ARGUMENT,
               "%s: layer %d has a null norm weight", what, l);
  }
  QG_REQUIRE(c.layers == 0 || (k_cache && v_cache && aligned(k_cache, 16) && aligned(v_cache, 16)),
             QG_ERR_INVALID_ARGUMENT, "%s: k_cache/v_cache NULL or misaligned", what);
  QG_REQUIRE(tokens && aligned(tokens, 4), QG_ERR_INVALID_ARGUMENT, "%s: tokens", what);
  QG_REQUIRE(!logits || aligned(logits, 4), QG_ERR_MISALIGNED, "%s: logits misaligned", what);
  const PrefillLayout Ly = prefill_layout(c, T);
  QG_REQUIRE(ws && ws_bytes >= Ly.total, QG_ERR_WORKSPACE_TOO_SMALL,
             "%s: workspace of %zu bytes given, %zu needed", what, ws_bytes, Ly.total);
  QG_REQUIRE(aligned(ws, 256), QG_ERR_MISALIGNED, "%s: ws not 256-byte aligned", what);

  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  float* x = reinterpret_cast<float*>(base + Ly.x);
  uint16_t* xn = reinterpret_cast<uint16_t*>(base + Ly.xn);
  float* q = reinterpret_cast<float*>(base + Ly.q);
  float* k = reinterpret_cast<float*>(base + Ly.k);
  float* v = reinterpret_cast<float*>(base + Ly.v);
  uint16_t* qb = reinterpret_cast<uint16_t*>(base + Ly.qb);
  uint16_t* att = reinterpret_cast<uint16_t*>(base + Ly.att);
  float* xa = reinterpret_cast<float*>(base + Ly.xa);
  uint16_t* xn2 = reinterpret_cast<uint16_t*>(base + Ly.xn2);
  float* gate = reinterpret_cast<float*>(base + Ly.gate);
  float* up = reinterpret_cast<float*>(base + Ly.up);
  uint16_t* hm = reinterpret_cast<uint16_t*>(base + Ly.h);
  unsigned* err = reinterpret_cast<unsigned*>(base + Ly.err);
  cudaMemsetAsync(err, 0, 4, s);

  const int H = c.heads, Hkv = c.kv_heads, D = c.head_dim, HD = H * D, KD = Hkv * D;
  const size_t layer_cache = (size_t)Hkv * cap * D;  // one sequence
  if ((st = qg_embed_affine8_g64(w->embed.w, w->embed.scales, w->embed.biases, tokens, x, c.vocab,
                                 c.hidden, T, stream)) != QG_OK)
    return st;
  clear_error();
  for (int l = 0; l < c.layers; ++l) {
    const qg_qwen3_layer& L = w->layers[l];
    uint16_t* kc = k_cache + l * layer_cache;
    uint16_t* vc = v_cache + l * layer_cache;
    rmsnorm_launch(x, L.input_norm, c.eps, xn, true, T, c.hidden, s, false);
    const A8Seg qkv[3] = {{L.q.w, L.q.scales, L.q.biases, q, nullptr, HD, 0},
                          {L.k.w, L.k.scales, L.k.biases, k, nullptr, KD, 0},
                          {L.v.w, L.v.scales, L.v.biases, v, nullptr, KD, 0}};
    gemm_affine8_launch(qkv, 3, xn, T, c.hidden, err, s, false, nullptr);
    launch_pdl(prefill_qk_kernel, dim3(T, (H + 2 * Hkv + 7) / 8), dim3(256), 0, s, false,
               (const float*)q, (const float*)k, (const float*)v, L.q_norm, L.k_norm, tokens,
               c.vocab, c.eps, c.theta, p0, qb, kc, vc, H, Hkv, D, cap);
    ar::Params P = {};
    P.q = qb;
    P.k = kc;
    P.v = vc;
    P.o = att;
    P.q_ld = HD;
    P.q_hs = D;
    P.k_ld = D;
    P.k_hs = (long long)cap * D;
    P.o_ld = HD;
    P.o_hs = D;
    P.T = T;
    P.S = p0 + T;
    P.H = H;
    P.Hkv = Hkv;
    P.causal = 1;
    P.scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    attn_rows_launch(P, 1, D, s);
    const A8Seg o = {L.o.w, L.o.scales, L.o.biases, xa, x, c.hidden, 0};
    gemm_affine8_launch(&o, 1, att, T, HD, err, s, false, nullptr);
    rmsnorm_launch(xa, L.post_norm, c.eps, xn2, true, T, c.hidden, s, false);
    const A8Seg gu[2] = {{L.gate.w, L.gate.scales, L.gate.biases, gate, nullptr, c.ffn, 0},
                         {L.up.w, L.up.scales, L.up.biases, up, nullptr, c.ffn, 0}};
    gemm_affine8_launch(gu, 2, xn2, T, c.hidden, err, s, false, nullptr);
    if ((st = qg_silu_mul(gate, up, hm, QG_BF16, T * c.ffn, stream)) != QG_OK) return st;
    const A8Seg dn = {L.down.w, L.down.scales, L.down.biases, x, xa, c.hidden, 0};
    gemm_affine8_launch(&dn, 1, hm, T, c.ffn, err, s, false, nullptr);
  }
  if (logits) {
    // the last row: final RMSNorm and the tied LM head
    const float* xl = x + (size_t)(T - 1) * c.hidden;
    GemvSeg h = {w->embed.w, w->embed.scales, w->embed.biases, logits, nullptr, c.vocab, 0};
    if (gemv_tc_eligible(&h, 1, c.hidden, 1, false)) {
      gemv_tc_launch_rmsnorm(&h, 1, xl, w->final_norm, c.eps, c.hidden, 1, s, false);
    } else {
      rmsnorm_launch(xl, w->final_norm, c.eps, xn, true, 1, c.hidden, s, false);
      gemv_affine8_launch(&h, 1, xn, false, c.hidden, 1, s, false);
    }
  }
  return check_launch(what);
}
